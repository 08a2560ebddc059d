// RoPE + position interpolation stage (HBM-bound).
//
// For every token m (original order) the pair (2i, 2i+1) of each q and k head vector is
// rotated by phi = (m / s) * base^(-2i/d) ("LoRA for Long-Context Adaptation", sections on
// RoPE and on position interpolation; interleaved pairs as in RoFormer). The rotated
// tensors are written head-major, [B][H][N][d], still in ORIGINAL token order: the -G/2
// roll of the shifted heads is never materialised, the attention kernels fold it into
// their row coordinates.
//
// Two kernels. The first computes the (cos, sin) table once per call, [N][d/2], in fp64
// (sincos of the exact angle at the start of each run of tokens, the angle-addition
// formulas along it), rounded to fp32; the backward's inverse
// rotation reads the same table from the workspace. The second streams q and k in 16-byte
// vectors, one CTA per token, and reads the token's table row (shared by all its heads,
// an L1/L2 hit) next to each vector: no CTA waits on fp64 arithmetic.
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

// (cos, sin) of (m / s) * base^(-2i/d) for every token m and pair i. The first kernel of
// every forward and of every backward that rotates: it also resets the status word and the
// persistent kernels' work counters, and records which arguments the rotation belongs to.
// A thread takes one pair i and a run of kTableRun consecutive tokens: the run's first angle
// in fp64 (pow, sincos), each next token by turning (cos, sin) through the step theta_i / s
// with the angle-addition formulas, in fp64. Over a run that drifts by about 1e-15, far
// below the fp32 rounding of the entries, at a fraction of a pow and a sincos per entry.
constexpr int kTableRun = 16;
__global__ void __launch_bounds__(256) rope_table_kernel(Params p) {
  const int half = p.d / 2;
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    for (int c = 0; c <= kNumWorkCounters; c++) p.status[c] = 0u;
    p.status[kFingerprintWord] = (unsigned)p.fingerprint;
    p.status[kFingerprintWord + 1] = (unsigned)(p.fingerprint >> 32);
  }
  const long runs = (long)((p.N + kTableRun - 1) / kTableRun) * half;
  const long stride = (long)gridDim.x * blockDim.x;
  for (long e = (long)blockIdx.x * blockDim.x + threadIdx.x; e < runs; e += stride) {
    const int i = (int)(e % half);                  // consecutive threads: consecutive pairs
    const int n0 = (int)(e / half) * kTableRun;
    const int n1 = min(n0 + kTableRun, p.N);
    const double theta = pow((double)p.rope_base, -2.0 * (double)i / (double)p.d);
    double ss, cs_step, sn, c;
    sincos(theta / (double)p.pi_scale, &ss, &cs_step);
    sincos(((double)n0 / (double)p.pi_scale) * theta, &sn, &c);
    float2* dst = p.cs + (size_t)n0 * half + i;
    for (int n = n0; n < n1; n++, dst += half) {
      *dst = make_float2((float)c, (float)sn);
      const double c_next = fma(c, cs_step, -sn * ss);
      sn = fma(sn, cs_step, c * ss);
      c = c_next;
    }
  }
}

// The loads of a token's q and k vectors are issued first (kBatch per thread in flight),
// then each vector is rotated with its four (or two) table entries and stored.
template <typename T>
__global__ void __launch_bounds__(256) rope_pi_kernel(Params p) {
  constexpr int V = 16 / sizeof(T);
  constexpr int kBatch = 4;
  const int tok = blockIdx.x;
  const int b = tok / p.N, n = tok - b * p.N;
  const uint4* q = reinterpret_cast<const uint4*>(static_cast<const T*>(p.q) +
                                                  (size_t)tok * p.Hq * p.d);
  const uint4* k = reinterpret_cast<const uint4*>(static_cast<const T*>(p.k) +
                                                  (size_t)tok * p.Hkv * p.d);
  const float2* cs_row = p.cs + (size_t)n * (p.d / 2);
  T* qr = static_cast<T*>(p.qr);
  T* kr = static_cast<T*>(p.kr);
  const int vq = p.Hq * p.d / V, vk = p.Hkv * p.d / V, nv = vq + vk;

  uint4 raw[kBatch];
#pragma unroll
  for (int u = 0; u < kBatch; u++) {
    const int e = threadIdx.x + u * blockDim.x;
    if (e < nv) raw[u] = __ldcs(e < vq ? q + e : k + (e - vq));
  }
  for (int e0 = threadIdx.x;; e0 += kBatch * blockDim.x) {
#pragma unroll
    for (int u = 0; u < kBatch; u++) {
      const int e = e0 + u * blockDim.x;
      if (e < nv) {
        const bool is_q = e < vq;
        const int ee = is_q ? e : e - vq;
        const int h = ee * V / p.d, c0 = ee * V - h * p.d;
        const int H = is_q ? p.Hq : p.Hkv;
        float2 cs[V / 2];
        const float4* c4 = reinterpret_cast<const float4*>(cs_row + c0 / 2);  // 16-B aligned
#pragma unroll
        for (int t = 0; t < V / 4; t++) {
          const float4 v = __ldg(c4 + t);
          cs[2 * t] = make_float2(v.x, v.y);
          cs[2 * t + 1] = make_float2(v.z, v.w);
        }
        T* dst = (is_q ? qr : kr) + (((size_t)b * H + h) * p.N + n) * p.d + c0;
        *reinterpret_cast<uint4*>(dst) = rotate_vec<T>(raw[u], cs);
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

cudaError_t launch_rope_table(const Params& p, cudaStream_t st) {
  const long runs = (long)((p.N + kTableRun - 1) / kTableRun) * (p.d / 2);
  long blocks = (runs + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  rope_table_kernel<<<dim3((unsigned)blocks), dim3(256), 0, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_rope_pi(const Params& p, bool bf16, cudaStream_t st) {
  dim3 grid(p.B * p.N), block(256);
  if (bf16)
    rope_pi_kernel<__nv_bfloat16><<<grid, block, 0, st>>>(p);
  else
    rope_pi_kernel<float><<<grid, block, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace s2
