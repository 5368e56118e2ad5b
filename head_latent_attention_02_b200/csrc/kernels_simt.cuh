// kernels_simt.cuh -- CUDA-core kernels: query absorption + RoPE relocation,
// the generic-dimension decode (fp32 or bf16 storage, fp32 arithmetic), the
// log-sum-exp merge and the value / output projections.
#pragma once
#include "common.cuh"

namespace mla {

// ---------------------------------------------------------------------------
// Absorption: q_abs[v, q, h, :d_c] = W_UK[h]^T q_nope[q, h]  (tutorial "Move
// the Key Projection Into the Query"); q_abs[v, q, h, d_c:] = R(q_pos[q] -
// delta[v]) q_rope[q, h] (RedKnot-MLA abstract: query-side RoPE relocation).
// grid (H, ceil(n_q / kAbsQ)), 256 threads.
constexpr int kAbsQ = 8;

struct AbsorbArgs {
  int n_q, H, d_c, d_r, d_n, n_ver;
  double rope_base;
  int delta[kMaxVersions];
  const void* q_nope;
  const void* q_rope;
  const int32_t* q_pos;
  const void* w_uk;
  void* q_abs;
};

template <typename T>
__global__ void __launch_bounds__(256) absorb_kernel(AbsorbArgs a) {
  extern __shared__ float sm_abs[];
  const int h = blockIdx.x;
  const int q0 = blockIdx.y * kAbsQ;
  const int nq = min(kAbsQ, a.n_q - q0);
  const int row = a.d_c + a.d_r;
  const T* qn = static_cast<const T*>(a.q_nope);
  const T* qr = static_cast<const T*>(a.q_rope);
  const T* w = static_cast<const T*>(a.w_uk) + (size_t)h * a.d_n * a.d_c;
  T* out = static_cast<T*>(a.q_abs);

  float* qs = sm_abs;  // [kAbsQ][d_n]
  for (int i = threadIdx.x; i < nq * a.d_n; i += blockDim.x) {
    const int qq = i / a.d_n, k = i % a.d_n;
    qs[qq * a.d_n + k] = to_f(qn[((size_t)(q0 + qq) * a.H + h) * a.d_n + k]);
  }
  __syncthreads();

  for (int c = threadIdx.x; c < a.d_c; c += blockDim.x) {
    float acc[kAbsQ];
#pragma unroll
    for (int qq = 0; qq < kAbsQ; ++qq) acc[qq] = 0.f;
    for (int k = 0; k < a.d_n; ++k) {
      const float wv = to_f(w[(size_t)k * a.d_c + c]);
#pragma unroll
      for (int qq = 0; qq < kAbsQ; ++qq) acc[qq] = fmaf(qs[qq * a.d_n + k], wv, acc[qq]);
    }
    for (int qq = 0; qq < nq; ++qq)
      for (int v = 0; v < a.n_ver; ++v)
        out[(((size_t)v * a.n_q + q0 + qq) * a.H + h) * row + c] = from_f<T>(acc[qq]);
  }

  // rotary part: pair i of the vector is rotated by (q_pos - delta) * theta_i,
  // theta_i = base^(-2i/d_r); angles in double precision
  const int half = a.d_r / 2;
  for (int t = threadIdx.x; t < nq * a.n_ver * half; t += blockDim.x) {
    const int i = t % half;
    const int v = (t / half) % a.n_ver;
    const int qq = t / (half * a.n_ver);
    const int q = q0 + qq;
    const double theta = pow(a.rope_base, -2.0 * i / a.d_r);
    const double ang = (double)(a.q_pos[q] - a.delta[v]) * theta;
    double sn, cs;
    sincos(ang, &sn, &cs);
    const size_t src = ((size_t)q * a.H + h) * a.d_r + 2 * i;
    const double x0 = to_f(qr[src]), x1 = to_f(qr[src + 1]);
    const size_t dst = (((size_t)v * a.n_q + q) * a.H + h) * row + a.d_c + 2 * i;
    out[dst] = from_f<T>((float)(x0 * cs - x1 * sn));
    out[dst + 1] = from_f<T>((float)(x0 * sn + x1 * cs));
  }
}

// ---------------------------------------------------------------------------
// Generic decode: one CTA per (head, query row), all of the sequence's rows,
// online softmax over chunks of 128 rows.  Any d_c, d_r; fp32 arithmetic.
// grid (n_h, n_q), 128 threads.
template <typename T>
__global__ void __launch_bounds__(128) decode_simt_kernel(DecodeArgs a) {
  extern __shared__ float sm_dec[];
  const int h = head_of(a, blockIdx.x);
  if (h < 0) return;
  const int qi = blockIdx.y;
  const int b = qi / a.s_q;
  const int row = a.d_c + a.d_r;
  const int tid = threadIdx.x;
  const T* qabs = static_cast<const T*>(a.q_abs);
  const T* cache = static_cast<const T*>(a.cache);

  float* qv = sm_dec;                       // [n_ver][row]
  float* acc = qv + a.n_ver * row;          // [d_c]
  float* pw = acc + a.d_c;                  // [128] weights of the chunk
  long long* prow = reinterpret_cast<long long*>(pw + 128);  // [128] physical rows
  float* red = reinterpret_cast<float*>(prow + 128);         // [4] reduction scratch

  for (int i = tid; i < a.n_ver * row; i += 128) {
    const int v = i / row, k = i % row;
    qv[i] = to_f(qabs[(((size_t)v * a.n_q + qi) * a.H + h) * row + k]);
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
          const T* r = cache + phys * row;
          const float* q = qv + ver * row;
          float d = 0.f;
          for (int k = 0; k < row; ++k) d = fmaf(q[k], to_f(r[k]), d);
          s = d * a.scale;
          if (a.key_inv) s *= a.key_inv[phys];
        }
      } else {
        phys = -1;
      }
    }
    // chunk max
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
        for (int t = 0; t < 128; ++t) {
          const long long pr = prow[t];
          if (pr >= 0) o = fmaf(pw[t], to_f(cache[pr * row + c]), o);
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
  for (int c = tid; c < a.d_c; c += 128) a.o_lat[orow * a.d_c + c] = empty ? 0.f : acc[c] * inv;
  if (tid == 0) a.lse[orow] = empty ? kNegInf : m_run + logf(l_run);
}

// ---------------------------------------------------------------------------
// Gather of the listed heads' absorbed queries into a dense block:
// q_pack[v, q, k, :] = q_abs[v, q, head_ids[k], :], so the tensor-core decode
// loads a block of heads with one box whatever the list.  One warp per packed
// row, 16-byte copies (row_bytes is a multiple of 16); an invalid id gives a
// zero row, whose results the decode does not write.  256 threads per block.
__global__ void __launch_bounds__(256) pack_heads_kernel(int rows_out, int n_h, int H,
                                                         int row_bytes, const int32_t* head_ids,
                                                         const uint8_t* q_abs, uint8_t* q_pack) {
  const int r = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= rows_out) return;
  const int vq = r / n_h, k = r % n_h;
  const int h = __ldg(head_ids + k);
  const int n16 = row_bytes / 16;
  uint4* dst = reinterpret_cast<uint4*>(q_pack + (size_t)r * row_bytes);
  if (h < 0 || h >= H) {
    for (int i = lane; i < n16; i += 32) dst[i] = make_uint4(0u, 0u, 0u, 0u);
    return;
  }
  const uint4* src = reinterpret_cast<const uint4*>(q_abs + ((size_t)vq * H + h) * row_bytes);
  for (int i = lane; i < n16; i += 32) dst[i] = __ldg(src + i);
}

// ---------------------------------------------------------------------------
// Log-sum-exp merge of two partial attentions (RedKnot-MLA abstract: offline
// and online paths merged before the shared output projection).  One warp per
// (query row, listed head); every lane reads both lse values before lane 0
// writes the merged one, so lse may alias lse_a or lse_b.  head_ids [n_h]
// names the heads (null: 0..n_h-1).  256 threads per block.
__global__ void __launch_bounds__(256) merge_lse_kernel(int n_q, int H, const int32_t* head_ids,
                                                        int n_h, int d,
                                                        const float* o_a, const float* lse_a,
                                                        const float* o_b, const float* lse_b,
                                                        float* o, float* lse) {
  const long long wid = blockIdx.x * 8ll + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (wid >= (long long)n_q * n_h) return;
  const int q = (int)(wid / n_h), hh = (int)(wid % n_h);
  const int h = head_ids ? __ldg(head_ids + hh) : hh;
  if (h < 0 || h >= H) {
    if (lane == 0) set_status(MLA_ERR_BAD_INDEX);
    return;
  }
  const size_t r = (size_t)q * H + h;
  const float la = lse_a[r], lb = lse_b[r];
  const float m = fmaxf(la, lb);
  float wa = 0.f, wb = 0.f, out_l = kNegInf;
  if (m != kNegInf) {
    wa = expf(la - m);
    wb = expf(lb - m);
    const float tot = wa + wb;
    out_l = m + logf(tot);
    wa /= tot;
    wb /= tot;
  }
  for (int c = lane; c < d; c += 32) {
    const float xa = (wa != 0.f) ? wa * o_a[r * d + c] : 0.f;
    const float xb = (wb != 0.f) ? wb * o_b[r * d + c] : 0.f;
    o[r * d + c] = xa + xb;
  }
  __syncwarp();
  if (lane == 0) lse[r] = out_l;
}

// ---------------------------------------------------------------------------
// v[q, h, :] = W_UV[h] o_lat[q, h, :]  (tutorial "Move the Value Expansion
// After the Weighted Sum").  grid (H, ceil(d_v / 8)), 256 threads (a warp per
// output feature, all query rows).  For bf16 storage the float activation is
// rounded to bf16 first, as the tensor-core product does.
template <typename T>
__global__ void __launch_bounds__(256) vproj_simt_kernel(int n_q, int H, int d_c, int d_v,
                                                         const float* o_lat, const T* w_uv,
                                                         float* v) {
  const int h = blockIdx.x;
  const int d = blockIdx.y * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (d >= d_v) return;
  const T* w = w_uv + ((size_t)h * d_v + d) * d_c;
  for (int q = 0; q < n_q; ++q) {
    const float* x = o_lat + ((size_t)q * H + h) * d_c;
    float acc = 0.f;
    for (int c = lane; c < d_c; c += 32) {
      float xv = x[c];
      if (sizeof(T) == 2) xv = round_bf16(xv);
      acc = fmaf(to_f(w[c]), xv, acc);
    }
    for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) v[((size_t)q * H + h) * d_v + d] = acc;
  }
}

// out[q, m] = W_O[m, :] . v[q, :]; a warp per output feature.  grid
// ceil(d_model / 8), 256 threads.
template <typename T>
__global__ void __launch_bounds__(256) oproj_simt_kernel(int n_q, int K, int d_model,
                                                         const float* v, const T* w_o,
                                                         float* out) {
  const int m = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (m >= d_model) return;
  const T* w = w_o + (size_t)m * K;
  for (int q = 0; q < n_q; ++q) {
    const float* x = v + (size_t)q * K;
    float acc = 0.f;
    for (int k = lane; k < K; k += 32) {
      float xv = x[k];
      if (sizeof(T) == 2) xv = round_bf16(xv);
      acc = fmaf(to_f(w[k]), xv, acc);
    }
    for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) out[(size_t)q * d_model + m] = acc;
  }
}

}  // namespace mla
