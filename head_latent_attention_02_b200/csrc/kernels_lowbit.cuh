// kernels_lowbit.cuh -- decode over a low-bit latent cache (QuantMLA abstract:
// the content and rotary caches stored as INT4 / INT4 or INT2 / INT4 codes,
// unpacked and dequantised inside the attention kernel).
//
// Each cached row is d_c content codes of bits_c bits, then d_r rotary codes
// of bits_r bits, packed little-end first (code k of a segment in bits
// [bits * k mod 8, ...) of byte bits * k / 8), two's complement fields.  With
// one static scale per channel, the score against the dequantised row is
// the score of the scale-multiplied query against the integer codes, and the
// weighted sum of dequantised latents is the weighted sum of codes times the
// content scale:
//   s_t = scale * ((q_c * sc) . code_c(t) + (q_r * sr) . code_r(t))
//   o   = (sum_t a_t code_c(t)) * sc
// so the kernel folds the scales into the query it keeps in shared memory
// and into the output, and works on codes otherwise.
//
// SIMT kernel, one CTA per (listed head, query row), 128 threads, the
// sequence's rows in chunks of 128 (one row per thread for the score, one
// channel per thread for the weighted sum), fp32 arithmetic throughout.
#pragma once
#include "common.cuh"

namespace mla {

// Quantisation of cache rows to packed codes: code = round-half-even(x /
// scale) clamped to the signed range, computed in fp32; the row's bytes are
// written whole.  One warp per row; lane l builds 32-bit words l, l + 32, ...
template <typename T, int BC, int BR>
__global__ void __launch_bounds__(256) pack_rows_kernel(int n_rows, int d_c, int d_r,
                                                        const T* rows, const float* scale_c,
                                                        const float* scale_r, uint8_t* out) {
  const int r = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= n_rows) return;
  const int width = d_c + d_r;
  const T* x = rows + (size_t)r * width;
  const int cwords = d_c * BC / 32, rwords = d_r * BR / 32;
  uint32_t* dst = reinterpret_cast<uint32_t*>(out + (size_t)r * (cwords + rwords) * 4);
  for (int w = lane; w < cwords + rwords; w += 32) {
    const bool content = w < cwords;
    const int bits = content ? BC : BR;
    const int per = 32 / bits;
    const int k0 = content ? w * per : (w - cwords) * per;
    const int lo = -(1 << (bits - 1)), hi = (1 << (bits - 1)) - 1;
    uint32_t word = 0;
    for (int j = 0; j < per; ++j) {
      const int k = k0 + j;
      const float v = content ? to_f(x[k]) / scale_c[k] : to_f(x[d_c + k]) / scale_r[k];
      const int code = min(hi, max(lo, (int)rintf(v)));
      word |= ((uint32_t)code & ((1u << bits) - 1u)) << (bits * j);
    }
    dst[w] = word;
  }
}

// signed code j of a 32-bit word of b-bit fields
template <int B>
__device__ __forceinline__ int code_of(uint32_t w, int j) {
  const uint32_t f = (w >> (B * j)) & ((1u << B) - 1u);
  const int sign = 1 << (B - 1);
  return (int)(f ^ sign) - sign;
}

// grid (n_h, n_q), 128 threads; dynamic shared memory as decode_simt_kernel.
template <typename T, int BC, int BR>
__global__ void __launch_bounds__(128) decode_lowbit_kernel(DecodeArgs a, const float* scale_c,
                                                            const float* scale_r) {
  extern __shared__ float sm_low[];
  const int h = head_of(a, blockIdx.x);
  if (h < 0) return;
  const int qi = blockIdx.y;
  const int b = qi / a.s_q;
  const int row = a.d_c + a.d_r;
  const int cwords = a.d_c * BC / 32, rwords = a.d_r * BR / 32;
  const int row_words = cwords + rwords;
  const int tid = threadIdx.x;
  const T* qabs = static_cast<const T*>(a.q_abs);
  const uint32_t* cache = static_cast<const uint32_t*>(a.cache);

  float* qv = sm_low;                       // [n_ver][row], channel scales folded in
  float* acc = qv + a.n_ver * row;          // [d_c] weighted sums of content codes
  float* pw = acc + a.d_c;                  // [128] weights of the chunk
  long long* prow = reinterpret_cast<long long*>(pw + 128);  // [128] physical rows
  float* red = reinterpret_cast<float*>(prow + 128);         // [4] reduction scratch

  for (int i = tid; i < a.n_ver * row; i += 128) {
    const int v = i / row, k = i % row;
    const float sc = k < a.d_c ? scale_c[k] : scale_r[k - a.d_c];
    qv[i] = to_f(qabs[(((size_t)v * a.n_q + qi) * a.qH + h) * row + k]) * sc;
  }
  for (int c = tid; c < a.d_c; c += 128) acc[c] = 0.f;
  __syncthreads();

  const int qp = a.q_pos[qi];
  const int n_att = attended_rows(a, b);
  float m_run = kNegInf, l_run = 0.f;
  for (int base = 0; base < n_att; base += 128) {
    const int i = base + tid;
    float s = kNegInf;
    long long phys = -1;
    if (i < n_att) {
      int kpos, ver;
      if (locate_row(a, b, i, &phys, &kpos, &ver)) {
        if (kpos <= qp) {
          const uint32_t* r = cache + phys * row_words;
          const float* q = qv + ver * row;
          float d = 0.f;
          for (int w = 0; w < cwords; ++w) {
            const uint32_t word = r[w];
#pragma unroll
            for (int j = 0; j < 32 / BC; ++j) d = fmaf(q[w * (32 / BC) + j], (float)code_of<BC>(word, j), d);
          }
          for (int w = 0; w < rwords; ++w) {
            const uint32_t word = r[cwords + w];
#pragma unroll
            for (int j = 0; j < 32 / BR; ++j)
              d = fmaf(q[a.d_c + w * (32 / BR) + j], (float)code_of<BR>(word, j), d);
          }
          s = d * a.scale;
        }
      } else {
        phys = -1;
      }
    }
    float mx = s;
    for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if ((tid & 31) == 0) red[tid >> 5] = mx;
    __syncthreads();
    mx = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
    __syncthreads();
    const float m_new = fmaxf(m_run, mx);
    float p = 0.f;
    if (s != kNegInf) p = expf(s - m_new);
    pw[tid] = p;
    prow[tid] = (p != 0.f) ? phys : -1;
    float sum = p;
    for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if ((tid & 31) == 0) red[tid >> 5] = sum;
    __syncthreads();
    sum = red[0] + red[1] + red[2] + red[3];
    const float corr = (m_run == kNegInf) ? 0.f : expf(m_run - m_new);
    if (m_new != kNegInf) {
      l_run = l_run * corr + sum;
      for (int c = tid; c < a.d_c; c += 128) {
        float o = acc[c] * corr;
        const int w = c / (32 / BC), j = c % (32 / BC);
        for (int t = 0; t < 128; ++t) {
          const long long pr = prow[t];
          if (pr >= 0) o = fmaf(pw[t], (float)code_of<BC>(cache[pr * row_words + w], j), o);
        }
        acc[c] = o;
      }
      m_run = m_new;
    }
    __syncthreads();
  }
  const size_t orow = ((size_t)qi * a.H + h);
  const bool empty = !(l_run > 0.f);
  const float inv = empty ? 0.f : 1.f / l_run;
  for (int c = tid; c < a.d_c; c += 128)
    a.o_lat[orow * a.d_c + c] = empty ? 0.f : acc[c] * inv * scale_c[c];
  if (tid == 0) a.lse[orow] = empty ? kNegInf : m_run + logf(l_run);
}

}  // namespace mla
