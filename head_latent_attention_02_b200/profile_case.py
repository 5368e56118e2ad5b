"""Small, self-contained launches of single kernels, sized for an ncu capture
(inputs above the 126 MB L2 where DRAM figures matter, a few hundred MB on
the device at most, three launches of the kernel).

    python -m head_latent_attention_02_b200.profile_case dequant

``dequant``: mla_dequant_rows over 65536 packed INT4/INT4 rows of the
512 + 64-channel latent (18.9 MB of codes in, 75.5 MB of bf16 rows out),
the pre-pass of the tensor-core low-bit decode at its 16 x 4096-row size.
"""
import sys

import torch

from . import build, mla
from .workloads import WORKLOADS


def dequant(n_rows: int = 65536) -> None:
    build.build()
    wl = WORKLOADS["bf16_b16_4k"]
    dims = mla.make_dims(wl)
    rb = (wl.d_c * 4 + wl.d_r * 4) // 8
    g = torch.Generator(device="cuda")
    g.manual_seed(1)
    packed = torch.randint(0, 256, (n_rows, rb), dtype=torch.uint8, device="cuda", generator=g)
    sc = torch.rand(wl.d_c, device="cuda", generator=g) + 0.5
    sr = torch.rand(wl.d_r, device="cuda", generator=g) + 0.5
    out = torch.empty((n_rows, wl.d_c + wl.d_r), dtype=torch.bfloat16, device="cuda")
    for _ in range(3):
        mla.dequant_rows(dims, 4, 4, packed, sc, sr, out)
    torch.cuda.synchronize()
    assert mla.get_status() == 0
    print("ok", float(out.float().abs().sum()))


CASES = {"dequant": dequant}

if __name__ == "__main__":
    if len(sys.argv) != 2 or sys.argv[1] not in CASES:
        sys.exit("usage: python -m head_latent_attention_02_b200.profile_case " + "|".join(CASES))
    CASES[sys.argv[1]]()
