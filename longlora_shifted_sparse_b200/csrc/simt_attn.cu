// CUDA-core S2-Attn kernels: the fp32 path and every shape the tensor-core path does not
// take (any even G, d a multiple of 32 up to 256), plus the backward's row-sum preprocess.
//
// One warp per row, lanes split the head dimension (lane owns elements lane + 32u). Rows
// are addressed in rolled coordinates: rolled row r of a shifted head is token
// (r + G/2) mod N, so the -G/2 roll and the +G/2 roll back are index arithmetic only
// ("LongLoRA: Efficient 100k Context LLM Fine-Tuning Guide", Implementation, Step 1,
// steps 3 and 5). Each group is attended on its own with the causal mask on group-local
// positions; the forward uses the online (running max / running sum) form of the
// max-subtracted softmax.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace s2 {

// Dot product of two lane-distributed rows, reduced over the warp (every lane gets it).
template <int DPL>
__device__ inline float row_dot(const float (&a)[DPL], const float (&b)[DPL]) {
  float acc = 0.f;
#pragma unroll
  for (int u = 0; u < DPL; u++) acc = fmaf(a[u], b[u], acc);
  return warp_sum(acc);
}

template <typename T, int DPL>
__device__ inline void load_row(const T* __restrict__ row, float (&x)[DPL], int lane) {
#pragma unroll
  for (int u = 0; u < DPL; u++) x[u] = to_f32<T>(row[lane + 32 * u]);
}

// Inverse rotation R(phi)^T of a lane-distributed row at token m (pair partner = lane ^ 1).
template <int DPL>
__device__ inline void inverse_rope(float (&x)[DPL], const float2* __restrict__ cs_row, int lane) {
#pragma unroll
  for (int u = 0; u < DPL; u++) {
    const int c = lane + 32 * u;
    const float partner = __shfl_xor_sync(0xffffffffu, x[u], 1);
    const float2 t = cs_row[c >> 1];
    // even c: x0 cos + x1 sin ; odd c: -x0 sin + x1 cos
    x[u] = (c & 1) ? fmaf(-partner, t.y, x[u] * t.x) : fmaf(x[u], t.x, partner * t.y);
  }
}

template <typename T, int DPL>
__global__ void __launch_bounds__(256) simt_fwd_kernel(Params p) {
  const int lane = threadIdx.x & 31;
  const long warp = ((long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (warp >= (long)p.B * p.Hq * p.N) return;
  const int r = (int)(warp % p.N);
  const int h = (int)((warp / p.N) % p.Hq);
  const int b = (int)(warp / ((long)p.N * p.Hq));
  const int kvh = h / (p.Hq / p.Hkv);
  const bool sh = q_head_shifted(h, p);
  const int g = r / p.G, i = r - g * p.G;
  const int m = src_row(r, sh, p.G, p.N);
  const int d = p.d;

  const T* qr = static_cast<const T*>(p.qr);
  const T* kr = static_cast<const T*>(p.kr);
  const T* v = static_cast<const T*>(p.v);
  float qv[DPL], acc[DPL], kv[DPL], vv[DPL];
  load_row<T, DPL>(qr + (((size_t)b * p.Hq + h) * p.N + m) * d, qv, lane);
#pragma unroll
  for (int u = 0; u < DPL; u++) acc[u] = 0.f;
  float mx = -INFINITY, l = 0.f;
  const int jend = p.causal ? i : p.G - 1;
  for (int j = 0; j <= jend; j++) {
    const int mj = src_row(g * p.G + j, sh, p.G, p.N);
    load_row<T, DPL>(kr + (((size_t)b * p.Hkv + kvh) * p.N + mj) * d, kv, lane);
    load_row<T, DPL>(v + (((size_t)b * p.N + mj) * p.Hkv + kvh) * d, vv, lane);
    const float s = row_dot<DPL>(qv, kv) * p.scale;
    const float mnew = fmaxf(mx, s);
    const float alpha = expf(mx - mnew);  // 0 on the first key (mx = -inf)
    const float pj = expf(s - mnew);
    l = fmaf(l, alpha, pj);
#pragma unroll
    for (int u = 0; u < DPL; u++) acc[u] = fmaf(acc[u], alpha, pj * vv[u]);
    mx = mnew;
  }
  const float inv_l = 1.f / l;
  T* o = static_cast<T*>(p.o) + (((size_t)b * p.N + m) * p.Hq + h) * d;
#pragma unroll
  for (int u = 0; u < DPL; u++) o[lane + 32 * u] = from_f32<T>(acc[u] * inv_l);
  if (lane == 0) p.lse[((size_t)b * p.Hq + h) * p.N + m] = mx + logf(l);
}

// The backward's first kernel when it reuses the forward's rotation: the call starts with a
// clean status word (no kernel of this launch reads it) and the work counters of the
// persistent kernels that follow at 0. With check_fingerprint, a workspace whose last
// rotation came from other arguments sets the stale bit, and the kernels that follow skip.
__device__ inline void backward_status_reset(const Params& p) {
  for (int c = 0; c <= kNumWorkCounters; c++) p.status[c] = 0u;
  if (p.check_fingerprint) {
    const unsigned long long f = (unsigned long long)p.status[kFingerprintWord] |
                                 ((unsigned long long)p.status[kFingerprintWord + 1] << 32);
    if (f != p.fingerprint) p.status[0] = kStatusStale;
  }
}

// D[b][h][m] = sum_c dO[b][m][h][c] * O[b][m][h][c] (fp32), one warp per row.
template <typename T, int DPL>
__global__ void __launch_bounds__(256) bwd_rowsum_kernel(Params p) {
  const int lane = threadIdx.x & 31;
  const long warp = ((long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (blockIdx.x == 0 && threadIdx.x == 0) backward_status_reset(p);
  if (warp >= (long)p.B * p.N * p.Hq) return;
  const int h = (int)(warp % p.Hq);
  const long bm = warp / p.Hq;
  const int m = (int)(bm % p.N), b = (int)(bm / p.N);
  const size_t off = (size_t)warp * p.d;
  float a[DPL], c[DPL];
  load_row<T, DPL>(static_cast<const T*>(p.dout) + off, a, lane);
  load_row<T, DPL>(static_cast<const T*>(p.o) + off, c, lane);
  const float D = row_dot<DPL>(a, c);
  if (lane == 0) p.Dsum[((size_t)b * p.Hq + h) * p.N + m] = D;
}

// D = rowsum(dO * O) for bf16 rows of 128 (the tensor-core path's shape), HBM-bound, plus
// the row terms of the tensor-core dK/dV pass. A CTA takes kRowsumTokens consecutive tokens
// of one batch entry with all their heads: those dO and O rows are contiguous in memory and
// are read front to back (a half-warp per 256-byte row, 16 bytes per lane, four rows of each
// tensor in flight per half-warp); the row sums go through shared memory and are written
// head by head, so that the LSE reads and the D and row-term writes are contiguous too.
constexpr int kRowsumTokens = 16;

__device__ inline void write_row_terms(const Params& p, size_t row, float D) {
  // -LSE*sqrt(d) and -D as sums of bf16 parts (each part the rounding of what the previous
  // ones left), exact to ~2^-24 and ~2^-16 relative
  const float nl = -p.lse[row] / p.scale;
  const __nv_bfloat16 l0 = __float2bfloat16_rn(nl);
  const float r1 = nl - __bfloat162float(l0);
  const __nv_bfloat16 l1 = __float2bfloat16_rn(r1);
  const __nv_bfloat16 l2 = __float2bfloat16_rn(r1 - __bfloat162float(l1));
  const __nv_bfloat16 d0 = __float2bfloat16_rn(-D);
  const __nv_bfloat16 d1 = __float2bfloat16_rn(-D - __bfloat162float(d0));
  const __nv_bfloat16 z = __float2bfloat16_rn(0.f);
  __nv_bfloat162 w[4] = {__halves2bfloat162(l0, l1), __halves2bfloat162(l2, d0),
                         __halves2bfloat162(d1, z), __halves2bfloat162(z, z)};
  uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.rowterms) + row * 16);
  dst[0] = *reinterpret_cast<const uint4*>(w);
  dst[1] = make_uint4(0u, 0u, 0u, 0u);
}

__global__ void __launch_bounds__(256) bwd_rowsum_bf16_d128_kernel(Params p) {
  extern __shared__ float dsh[];  // [kRowsumTokens][Hq]
  const int chunk = threadIdx.x & 15;                          // 16-byte piece of a row
  const int hw = threadIdx.x >> 4, nhw = blockDim.x >> 4;  // half-warp id and count
  if (blockIdx.x == 0 && threadIdx.x == 0) backward_status_reset(p);
  const int blocks_per_b = (p.N + kRowsumTokens - 1) / kRowsumTokens;
  const int b = blockIdx.x / blocks_per_b;
  const int m0 = (blockIdx.x - b * blocks_per_b) * kRowsumTokens;
  const int ntok = min(kRowsumTokens, p.N - m0);
  const int nrows = ntok * p.Hq;  // rows (token, head) of this CTA, contiguous in dO and O
  const uint4* dO = reinterpret_cast<const uint4*>(p.dout) + ((size_t)b * p.N + m0) * p.Hq * 16;
  const uint4* O = reinterpret_cast<const uint4*>(p.o) + ((size_t)b * p.N + m0) * p.Hq * 16;
  for (int r0 = hw; r0 < nrows; r0 += 4 * nhw) {
    uint4 a[4], c[4];
#pragma unroll
    for (int i = 0; i < 4; i++) {
      const int r = r0 + i * nhw;
      const size_t e = r < nrows ? (size_t)r * 16 + chunk : 0;
      a[i] = __ldcs(dO + e);
      c[i] = __ldcs(O + e);
    }
#pragma unroll
    for (int i = 0; i < 4; i++) {
      const __nv_bfloat162* x = reinterpret_cast<const __nv_bfloat162*>(&a[i]);
      const __nv_bfloat162* y = reinterpret_cast<const __nv_bfloat162*>(&c[i]);
      float acc = 0.f;
#pragma unroll
      for (int t = 0; t < 4; t++) {
        const float2 xf = __bfloat1622float2(x[t]), yf = __bfloat1622float2(y[t]);
        acc = fmaf(xf.x, yf.x, acc);
        acc = fmaf(xf.y, yf.y, acc);
      }
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      const int r = r0 + i * nhw;
      if (chunk == 0 && r < nrows) dsh[r] = acc;  // [token][head]
    }
  }
  __syncthreads();
  // head by head: consecutive threads take consecutive tokens of one head
  for (int e = threadIdx.x; e < nrows; e += blockDim.x) {
    const int h = e / ntok, t = e - h * ntok;
    const size_t row = ((size_t)b * p.Hq + h) * p.N + m0 + t;
    const float D = dsh[t * p.Hq + h];
    p.Dsum[row] = D;
    write_row_terms(p, row, D);
  }
}

template <typename T, int DPL>
__global__ void __launch_bounds__(256) simt_dq_kernel(Params p) {
  const int lane = threadIdx.x & 31;
  const long warp = ((long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (warp >= (long)p.B * p.Hq * p.N) return;
  const int r = (int)(warp % p.N);
  const int h = (int)((warp / p.N) % p.Hq);
  const int b = (int)(warp / ((long)p.N * p.Hq));
  const int kvh = h / (p.Hq / p.Hkv);
  const bool sh = q_head_shifted(h, p);
  const int g = r / p.G, i = r - g * p.G;
  const int m = src_row(r, sh, p.G, p.N);
  const int d = p.d;

  const T* qr = static_cast<const T*>(p.qr);
  const T* kr = static_cast<const T*>(p.kr);
  const T* v = static_cast<const T*>(p.v);
  float qv[DPL], dov[DPL], dq[DPL], kv[DPL], vv[DPL];
  load_row<T, DPL>(qr + (((size_t)b * p.Hq + h) * p.N + m) * d, qv, lane);
  load_row<T, DPL>(static_cast<const T*>(p.dout) + (((size_t)b * p.N + m) * p.Hq + h) * d, dov,
                   lane);
  const float lse = p.lse[((size_t)b * p.Hq + h) * p.N + m];
  const float Dm = p.Dsum[((size_t)b * p.Hq + h) * p.N + m];
#pragma unroll
  for (int u = 0; u < DPL; u++) dq[u] = 0.f;
  const int jend = p.causal ? i : p.G - 1;
  for (int j = 0; j <= jend; j++) {
    const int mj = src_row(g * p.G + j, sh, p.G, p.N);
    load_row<T, DPL>(kr + (((size_t)b * p.Hkv + kvh) * p.N + mj) * d, kv, lane);
    load_row<T, DPL>(v + (((size_t)b * p.N + mj) * p.Hkv + kvh) * d, vv, lane);
    const float s = row_dot<DPL>(qv, kv) * p.scale;
    const float pr = expf(s - lse);
    const float dp = row_dot<DPL>(dov, vv);
    const float ds = pr * (dp - Dm);
#pragma unroll
    for (int u = 0; u < DPL; u++) dq[u] = fmaf(ds, kv[u], dq[u]);
  }
#pragma unroll
  for (int u = 0; u < DPL; u++) dq[u] *= p.scale;
  inverse_rope<DPL>(dq, p.cs + (size_t)m * (d / 2), lane);
  T* out = static_cast<T*>(p.dq) + (((size_t)b * p.N + m) * p.Hq + h) * d;
#pragma unroll
  for (int u = 0; u < DPL; u++) out[lane + 32 * u] = from_f32<T>(dq[u]);
}

template <typename T, int DPL>
__global__ void __launch_bounds__(256) simt_dkdv_kernel(Params p) {
  const int lane = threadIdx.x & 31;
  const long warp = ((long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (warp >= (long)p.B * p.Hkv * p.N) return;
  const int r = (int)(warp % p.N);
  const int kvh = (int)((warp / p.N) % p.Hkv);
  const int b = (int)(warp / ((long)p.N * p.Hkv));
  const int R = p.Hq / p.Hkv;
  const bool sh = kv_head_shifted(kvh, p);
  const int g = r / p.G, j = r - g * p.G;
  const int m = src_row(r, sh, p.G, p.N);
  const int d = p.d;

  const T* qr = static_cast<const T*>(p.qr);
  const T* kr = static_cast<const T*>(p.kr);
  const T* dout = static_cast<const T*>(p.dout);
  float kv[DPL], vv[DPL], dk[DPL], dv[DPL], qv[DPL], dov[DPL];
  load_row<T, DPL>(kr + (((size_t)b * p.Hkv + kvh) * p.N + m) * d, kv, lane);
  load_row<T, DPL>(static_cast<const T*>(p.v) + (((size_t)b * p.N + m) * p.Hkv + kvh) * d, vv,
                   lane);
#pragma unroll
  for (int u = 0; u < DPL; u++) dk[u] = dv[u] = 0.f;
  const int ibeg = p.causal ? j : 0;
  for (int rr = 0; rr < R; rr++) {
    const int h = kvh * R + rr;
    for (int i = ibeg; i < p.G; i++) {
      const int mi = src_row(g * p.G + i, sh, p.G, p.N);
      load_row<T, DPL>(qr + (((size_t)b * p.Hq + h) * p.N + mi) * d, qv, lane);
      load_row<T, DPL>(dout + (((size_t)b * p.N + mi) * p.Hq + h) * d, dov, lane);
      const float lse = p.lse[((size_t)b * p.Hq + h) * p.N + mi];
      const float Dm = p.Dsum[((size_t)b * p.Hq + h) * p.N + mi];
      const float s = row_dot<DPL>(qv, kv) * p.scale;
      const float pr = expf(s - lse);
      const float dp = row_dot<DPL>(dov, vv);
      const float ds = pr * (dp - Dm);
#pragma unroll
      for (int u = 0; u < DPL; u++) {
        dv[u] = fmaf(pr, dov[u], dv[u]);
        dk[u] = fmaf(ds, qv[u], dk[u]);
      }
    }
  }
#pragma unroll
  for (int u = 0; u < DPL; u++) dk[u] *= p.scale;
  inverse_rope<DPL>(dk, p.cs + (size_t)m * (d / 2), lane);
  const size_t off = (((size_t)b * p.N + m) * p.Hkv + kvh) * d;
  T* dko = static_cast<T*>(p.dk) + off;
  T* dvo = static_cast<T*>(p.dv) + off;
#pragma unroll
  for (int u = 0; u < DPL; u++) {
    dko[lane + 32 * u] = from_f32<T>(dk[u]);
    dvo[lane + 32 * u] = from_f32<T>(dv[u]);
  }
}

namespace {
constexpr int kWarpsPerBlock = 8;

inline dim3 warp_grid(long rows) {
  return dim3((unsigned)((rows + kWarpsPerBlock - 1) / kWarpsPerBlock));
}
}  // namespace

#define S2_DISPATCH_DPL(KERNEL, T, DPL_RT, GRID, ST, P)                          \
  switch (DPL_RT) {                                                              \
    case 1: KERNEL<T, 1><<<GRID, kWarpsPerBlock * 32, 0, ST>>>(P); break;        \
    case 2: KERNEL<T, 2><<<GRID, kWarpsPerBlock * 32, 0, ST>>>(P); break;        \
    case 3: KERNEL<T, 3><<<GRID, kWarpsPerBlock * 32, 0, ST>>>(P); break;        \
    case 4: KERNEL<T, 4><<<GRID, kWarpsPerBlock * 32, 0, ST>>>(P); break;        \
    case 5: KERNEL<T, 5><<<GRID, kWarpsPerBlock * 32, 0, ST>>>(P); break;        \
    case 6: KERNEL<T, 6><<<GRID, kWarpsPerBlock * 32, 0, ST>>>(P); break;        \
    case 7: KERNEL<T, 7><<<GRID, kWarpsPerBlock * 32, 0, ST>>>(P); break;        \
    case 8: KERNEL<T, 8><<<GRID, kWarpsPerBlock * 32, 0, ST>>>(P); break;        \
    default: return cudaErrorInvalidValue;                                       \
  }

#define S2_DISPATCH_TYPE(KERNEL, BF16, GRID, ST, P)                              \
  if (BF16) {                                                                    \
    S2_DISPATCH_DPL(KERNEL, __nv_bfloat16, (P).d / 32, GRID, ST, P)              \
  } else {                                                                       \
    S2_DISPATCH_DPL(KERNEL, float, (P).d / 32, GRID, ST, P)                      \
  }

cudaError_t launch_simt_fwd(const Params& p, bool bf16, cudaStream_t st) {
  dim3 grid = warp_grid((long)p.B * p.Hq * p.N);
  S2_DISPATCH_TYPE(simt_fwd_kernel, bf16, grid, st, p)
  return cudaGetLastError();
}

cudaError_t launch_bwd_rowsum(const Params& p, bool bf16, cudaStream_t st) {
  if (bf16 && p.d == 128) {
    const long blocks = (long)p.B * ((p.N + kRowsumTokens - 1) / kRowsumTokens);
    const size_t smem = (size_t)kRowsumTokens * p.Hq * sizeof(float);
    if (smem > 48 * 1024) {
      cudaError_t e = cudaFuncSetAttribute(bwd_rowsum_bf16_d128_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
    }
    bwd_rowsum_bf16_d128_kernel<<<(unsigned)blocks, 256, smem, st>>>(p);
    return cudaGetLastError();
  }
  dim3 grid = warp_grid((long)p.B * p.Hq * p.N);
  S2_DISPATCH_TYPE(bwd_rowsum_kernel, bf16, grid, st, p)
  return cudaGetLastError();
}

cudaError_t launch_simt_dq(const Params& p, bool bf16, cudaStream_t st) {
  dim3 grid = warp_grid((long)p.B * p.Hq * p.N);
  S2_DISPATCH_TYPE(simt_dq_kernel, bf16, grid, st, p)
  return cudaGetLastError();
}

cudaError_t launch_simt_dkdv(const Params& p, bool bf16, cudaStream_t st) {
  dim3 grid = warp_grid((long)p.B * p.Hkv * p.N);
  S2_DISPATCH_TYPE(simt_dkdv_kernel, bf16, grid, st, p)
  return cudaGetLastError();
}

}  // namespace s2
