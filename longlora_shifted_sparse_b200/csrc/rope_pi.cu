// RoPE + position interpolation stage (HBM-bound).
//
// For every token m (original order) the pair (2i, 2i+1) of each q and k head vector is
// rotated by phi = (m / s) * base^(-2i/d) ("LoRA for Long-Context Adaptation", sections on
// RoPE and on position interpolation; interleaved pairs as in RoFormer). The rotated
// tensors are written head-major, [B][H][N][d], still in ORIGINAL token order: the -G/2
// roll of the shifted heads is never materialised, the attention kernels fold it into
// their row coordinates.
//
// One CTA per token. The d/2 angles of a token are shared by all heads of q and k, so the
// CTA computes them once in fp64 (sincos of an exact fp64 angle, rounded to fp32) and
// keeps them in shared memory; the (cos, sin) table is also written to the workspace for
// the backward's inverse rotation. The data moves in 16-byte vectors.
#include "common.cuh"
#include "kernels.h"

namespace s2 {

template <typename T>
__device__ inline uint4 rotate_vec(uint4 raw, const float2* __restrict__ cs_row) {
  constexpr int V = 16 / sizeof(T);
  const T* x = reinterpret_cast<const T*>(&raw);
  uint4 out_raw;
  T* y = reinterpret_cast<T*>(&out_raw);
#pragma unroll
  for (int t = 0; t < V / 2; t++) {
    float2 c = cs_row[t];
    float x0 = to_f32<T>(x[2 * t]), x1 = to_f32<T>(x[2 * t + 1]);
    y[2 * t] = from_f32<T>(fmaf(x0, c.x, -x1 * c.y));
    y[2 * t + 1] = from_f32<T>(fmaf(x0, c.y, x1 * c.x));
  }
  return out_raw;
}

// The loads of a token's q and k vectors are issued first (kBatch per thread in flight),
// the fp64 angles are computed while they are in flight, then the vectors are rotated and
// stored: the kernel is bound by HBM, so it needs many loads outstanding per SM.
template <typename T>
__global__ void __launch_bounds__(256) rope_pi_kernel(Params p) {
  extern __shared__ float2 s_cs[];
  constexpr int V = 16 / sizeof(T);
  constexpr int kBatch = 4;
  const int half = p.d / 2;
  const int tok = blockIdx.x;
  const int b = tok / p.N, n = tok - b * p.N;
  if (tok == 0 && threadIdx.x == 0) {
    p.status[0] = 0u;  // each call starts with a clean status and work counters at 0
    for (int c = 1; c <= kNumWorkCounters; c++) p.status[c] = 0u;
  }

  const uint4* q = reinterpret_cast<const uint4*>(static_cast<const T*>(p.q) +
                                                  (size_t)tok * p.Hq * p.d);
  const uint4* k = reinterpret_cast<const uint4*>(static_cast<const T*>(p.k) +
                                                  (size_t)tok * p.Hkv * p.d);
  T* qr = static_cast<T*>(p.qr);
  T* kr = static_cast<T*>(p.kr);
  const int vq = p.Hq * p.d / V, vk = p.Hkv * p.d / V, nv = vq + vk;

  uint4 raw[kBatch];
#pragma unroll
  for (int u = 0; u < kBatch; u++) {
    const int e = threadIdx.x + u * blockDim.x;
    if (e < nv) raw[u] = __ldcs(e < vq ? q + e : k + (e - vq));
  }
  for (int i = threadIdx.x; i < half; i += blockDim.x) {
    double theta = pow((double)p.rope_base, -2.0 * (double)i / (double)p.d);
    double phi = ((double)n / (double)p.pi_scale) * theta;
    double sn, c;
    sincos(phi, &sn, &c);
    float2 v = make_float2((float)c, (float)sn);
    s_cs[i] = v;
    if (b == 0) p.cs[(size_t)n * half + i] = v;
  }
  __syncthreads();

  for (int e0 = threadIdx.x;; e0 += kBatch * blockDim.x) {
#pragma unroll
    for (int u = 0; u < kBatch; u++) {
      const int e = e0 + u * blockDim.x;
      if (e < nv) {
        const bool is_q = e < vq;
        const int ee = is_q ? e : e - vq;
        const int h = ee * V / p.d, c0 = ee * V - h * p.d;
        const int H = is_q ? p.Hq : p.Hkv;
        T* dst = (is_q ? qr : kr) + (((size_t)b * H + h) * p.N + n) * p.d + c0;
        *reinterpret_cast<uint4*>(dst) = rotate_vec<T>(raw[u], s_cs + c0 / 2);
      }
    }
    if (e0 + kBatch * (int)blockDim.x >= nv) break;
#pragma unroll
    for (int u = 0; u < kBatch; u++) {  // next batch (tokens with more than 1024 vectors)
      const int e = e0 + kBatch * blockDim.x + u * blockDim.x;
      if (e < nv) raw[u] = __ldcs(e < vq ? q + e : k + (e - vq));
    }
  }
}

cudaError_t launch_rope_pi(const Params& p, bool bf16, cudaStream_t st) {
  dim3 grid(p.B * p.N), block(256);
  size_t smem = (size_t)(p.d / 2) * sizeof(float2);
  if (bf16)
    rope_pi_kernel<__nv_bfloat16><<<grid, block, smem, st>>>(p);
  else
    rope_pi_kernel<float><<<grid, block, smem, st>>>(p);
  return cudaGetLastError();
}

}  // namespace s2
