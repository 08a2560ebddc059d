// S2-Attn backward on the tcgen05 tensor cores: a dK/dV pass and a dQ pass.
//
// Both passes recompute the probabilities from the forward's LSE instead of storing them:
// P = exp(S / sqrt(d) - LSE), dP = dO V^T, dS = P * (dP - D) with D = rowsum(dO * O) from
// the preprocess kernel. Rows are addressed exactly as in the forward: the tiles of a
// shifted head start at token (r0 + G/2) mod N, so the -G/2 roll and the +G/2 roll back
// are TMA row coordinates and store addresses ("LongLoRA and Shifted Sparse Attention
// (S^2-Attn)", definition; "LongLoRA: Efficient 100k Context LLM Fine-Tuning Guide",
// Implementation, Step 1). Gradients are taken with respect to the rotated q~, k~ and then
// rotated back, dq = R(phi)^T dq~, dk = R(phi)^T dk~ ("LoRA for Long-Context Adaptation",
// RoPE and position-interpolation sections), using the workspace's (cos, sin) table.
//
// Both passes walk the other side of the group in 64-row half tiles u = 0, 1, 2, ... with
// two TMEM score buffers, so the tensor cores compute half u+1 while the per-row math of
// half u runs. MMA issue order per half: scores of u+1, then the gradient MMAs of u.
//
// dK/dV pass: one CTA per 128-row key tile (b, kv head, group, kt). For every query head of
// the kv head and every query tile it >= kt (causal), in two 64-row halves:
//     S^T  = K Q_h^T     (SS MMA, N = 64)             thread = key row = TMEM lane
//     dP^T = V dO_h^T    (SS MMA, N = 64)
//     P^T  = exp2(S^T log2(e)/sqrt(d) - LSE_i log2(e)) -> bf16 over S^T
//     dS^T = P^T * (dP^T - D_i)                        -> bf16 over dP^T
//     dV  += P^T dO_h    (TS MMA, K = 64)
//     dK  += dS^T Q_h    (TS MMA, K = 64)
//   TMEM: S^T_0 [0,64) dP^T_0 [64,128) S^T_1 [128,192) dP^T_1 [192,256) dV [256,384)
//   dK [384,512). The GQA sum over query heads happens in the TMEM accumulators.
//   Epilogue: dk = R^T (dK / sqrt(d)), dv = dV, bf16, at the key tokens' original rows.
// dQ pass: one CTA per 128-row query tile (b, head, group, qt). For every key tile j <= qt,
//   in two 64-row halves: S = Q K_h^T, dP = dO V_h^T (SS MMAs, N = 64); dS = P (dP - D)
//   -> bf16 over S (thread = query row); dQ += dS K_h (TS MMA, K = 64).
//   TMEM: S_0 [0,64) dP_0 [64,128) S_1 [128,192) dP_1 [192,256) dQ [256,384).
//   Epilogue: dq = R^T (dQ / sqrt(d)), bf16, at the query tokens' original rows.
// CTAs are launched head-group-major so that the CTAs running together share the tiles
// they stream (L2 reuse). Roles as in the forward: warp 0 TMA producer, warp 1 MMA issuer
// and TMEM owner, warps 2..5 the per-row math. Every wait is bounded (see sm100.cuh).
#include "common.cuh"
#include "sm100.cuh"
#include "tc_kernels.h"
#include "tma_host.h"

namespace s2 {
namespace {

using namespace sm100;

constexpr int kD = 128;
constexpr int kTile = 128;
constexpr int kHalf = 64;                          // rows per half tile
constexpr uint32_t kTileBytes = kTile * kD * 2;
constexpr uint32_t kBoxBytes = kTileBytes / 2;     // one 128-row x 64-column TMA box
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// K-major operand starting at row `row0` (multiple of 8) of a 128 x 128 tile, k-step kk.
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t tile_saddr, int kk, int row0 = 0) {
  return smem_desc_sw128(tile_saddr + (kk >> 2) * kBoxBytes + (kk & 3) * 32 + row0 * 128, 16,
                         1024);
}

// Tile rows as an MN-major B operand (K = rows, N = d): k-step kk covers rows
// row0 + 16kk .. row0 + 16kk + 15.
__device__ __forceinline__ uint64_t mn_desc(uint32_t tile_saddr, int kk, int row0 = 0) {
  return smem_desc_sw128(tile_saddr + (row0 + kk * 16) * 128, kBoxBytes, 1024);
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

// Rotates a chunk of 32 consecutive fp32 columns (16 channel pairs starting at pair p0)
// back by R(phi)^T, scales it, and packs it to bf16.
__device__ __forceinline__ void unrotate_pack(const uint32_t (&x)[32], const float2* cs_row,
                                              int p0, float scale, uint4 (&out)[4]) {
  uint32_t* w = reinterpret_cast<uint32_t*>(out);
#pragma unroll
  for (int t = 0; t < 16; t++) {
    const float2 c = cs_row[p0 + t];
    const float x0 = __uint_as_float(x[2 * t]) * scale, x1 = __uint_as_float(x[2 * t + 1]) * scale;
    w[t] = pack_bf16x2(fmaf(x0, c.x, x1 * c.y), fmaf(-x0, c.y, x1 * c.x));
  }
}

__device__ __forceinline__ void scale_pack(const uint32_t (&x)[32], float scale, uint4 (&out)[4]) {
  uint32_t* w = reinterpret_cast<uint32_t*>(out);
#pragma unroll
  for (int t = 0; t < 16; t++)
    w[t] = pack_bf16x2(__uint_as_float(x[2 * t]) * scale, __uint_as_float(x[2 * t + 1]) * scale);
}

// ================================================================================ dK / dV

// smem: K | V | stage 0: Q, dO | stage 1: Q, dO | LSE[2][128] | D[2][128]
constexpr uint32_t kKVOffK = 0;
constexpr uint32_t kKVOffV = kTileBytes;
constexpr uint32_t kKVOffStage = 2 * kTileBytes;   // + s * 2 * kTileBytes: Q then dO
constexpr uint32_t kKVOffLse = 6 * kTileBytes;     // + s * 512
constexpr uint32_t kKVOffD = 6 * kTileBytes + 1024;
constexpr uint32_t kKVSmem = 6 * kTileBytes + 2048 + 1024;

struct DkdvBarriers {
  uint64_t kv_full;
  uint64_t q_full[2], q_empty[2];
  uint64_t sdp_full[2], p_ready[2], ds_ready[2];
  uint64_t acc_done, drain;
};

__global__ void __launch_bounds__(kThreads, 1)
    tc_dkdv_kernel(const Params p, const __grid_constant__ CUtensorMap tm_q,
                   const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                   const __grid_constant__ CUtensorMap tm_do) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  __shared__ DkdvBarriers bars;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = p.G / kTile, ng = p.N / p.G, R = p.Hq / p.Hkv;
  // head-group-major: the key tiles of one (b, kv head, group) run together, heaviest first
  const int kt = (int)(blockIdx.x % T);
  const int bkg = (int)(blockIdx.x / T);
  const int g = bkg % ng, bk = bkg / ng;
  const int kvh = bk % p.Hkv, b = bk / p.Hkv;
  const bool sh = head_shifted(kvh, p.Hkv);
  const int it0 = p.causal ? kt : 0;
  const int nq = T - it0;         // query tiles per query head
  const int ntiles = R * nq;      // (query head, query tile) pairs
  const int nsteps = 2 * ntiles;  // 64-row halves
  const int mk0 = src_row(g * p.G + kt * kTile, sh, p.G, p.N);

  Abort ab{&abort_flag, p.status};
  if (threadIdx.x == 0) {
    abort_flag = *reinterpret_cast<volatile unsigned*>(p.status) != 0u;
    mbar_init(smem_addr(&bars.kv_full), 1);
    for (int s = 0; s < 2; s++) {
      mbar_init(smem_addr(&bars.q_full[s]), 1);
      mbar_init(smem_addr(&bars.q_empty[s]), 1);
      mbar_init(smem_addr(&bars.sdp_full[s]), 1);
      mbar_init(smem_addr(&bars.p_ready[s]), 128);
      mbar_init(smem_addr(&bars.ds_ready[s]), 128);
    }
    mbar_init(smem_addr(&bars.acc_done), 1);
    mbar_init(smem_addr(&bars.drain), 1);
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(smem_addr(&tmem_base_sh), kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  const uint32_t colDV = 256, colDK = 384;
  const uint32_t sK = smem_addr(smem + kKVOffK), sV = smem_addr(smem + kKVOffV);
  const bool skip = abort_flag != 0;

  if (skip) {
  } else if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      const uint32_t kvb = smem_addr(&bars.kv_full);
      mbar_arrive_expect_tx(kvb, 2 * kTileBytes);
      const int krow = (b * p.Hkv + kvh) * p.N + mk0;
      tma_load_2d(sK, &tm_k, kvb, 0, krow);
      tma_load_2d(sK + kBoxBytes, &tm_k, kvb, 64, krow);
      tma_load_3d(sV, &tm_v, kvb, 0, kvh, b * p.N + mk0);
      tma_load_3d(sV + kBoxBytes, &tm_v, kvb, 64, kvh, b * p.N + mk0);
      int issued = 0;
      for (int n = 0; n < ntiles; n++) {
        const int s = n & 1;
        const uint32_t ph = (n >> 1) & 1;
        const int h = kvh * R + n / nq;
        const int it = it0 + n % nq;
        const int mq0 = src_row(g * p.G + it * kTile, sh, p.G, p.N);
        if (!mbar_wait(smem_addr(&bars.q_empty[s]), ph ^ 1, ab)) break;
        const uint32_t qb = smem_addr(&bars.q_full[s]);
        const uint32_t sQ = smem_addr(smem + kKVOffStage + s * 2 * kTileBytes);
        const uint32_t sDO = sQ + kTileBytes;
        mbar_arrive_expect_tx(qb, 2 * kTileBytes + 1024);
        const int qrow = (b * p.Hq + h) * p.N + mq0;
        tma_load_2d(sQ, &tm_q, qb, 0, qrow);
        tma_load_2d(sQ + kBoxBytes, &tm_q, qb, 64, qrow);
        tma_load_3d(sDO, &tm_do, qb, 0, h, b * p.N + mq0);
        tma_load_3d(sDO + kBoxBytes, &tm_do, qb, 64, h, b * p.N + mq0);
        const size_t lrow = ((size_t)b * p.Hq + h) * p.N + mq0;
        bulk_load(smem_addr(smem + kKVOffLse + s * 512), p.lse + lrow, 512, qb);
        bulk_load(smem_addr(smem + kKVOffD + s * 512), p.Dsum + lrow, 512, qb);
        issued = n + 1;
      }
      int no_abort = 0;
      Abort local{&no_abort, p.status};
      for (int n = issued - 1; n >= 0 && n >= issued - 2; n--)
        mbar_wait(smem_addr(&bars.q_full[n & 1]), (n >> 1) & 1, local);
      mbar_wait(kvb, 0, local);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16_f32(kTile, kHalf, false, false);
      const uint32_t idesc_g = idesc_bf16_f32(kTile, kD, false, true);
      bool ok = mbar_wait(smem_addr(&bars.kv_full), 0, ab);
      // scores of half u into buffer u & 1 (waits for its query tile on the first half)
      auto issue_scores = [&](int u) -> bool {
        const int n = u >> 1, hf = u & 1, s = n & 1;
        if (hf == 0 && !mbar_wait(smem_addr(&bars.q_full[s]), (n >> 1) & 1, ab)) return false;
        tc_fence_after();
        const uint32_t sQ = smem_addr(smem + kKVOffStage + s * 2 * kTileBytes);
        const uint32_t sDO = sQ + kTileBytes;
        const uint32_t cST = (u & 1) * 128, cDPT = cST + 64;
#pragma unroll
        for (int kk = 0; kk < kD / 16; kk++)
          mma_ss(tmem + cST, kmajor_desc(sK, kk), kmajor_desc(sQ, kk, hf * kHalf), idesc_s, kk > 0);
#pragma unroll
        for (int kk = 0; kk < kD / 16; kk++)
          mma_ss(tmem + cDPT, kmajor_desc(sV, kk), kmajor_desc(sDO, kk, hf * kHalf), idesc_s,
                 kk > 0);
        mma_commit(smem_addr(&bars.sdp_full[u & 1]));
        return true;
      };
      tc_fence_after();
      if (ok && nsteps > 0) ok = issue_scores(0);
      for (int u = 0; ok && u < nsteps; u++) {
        if (u + 1 < nsteps && !issue_scores(u + 1)) break;
        const int n = u >> 1, hf = u & 1, s = n & 1, bb = u & 1;
        const uint32_t ph = (u >> 1) & 1;
        const uint32_t sQ = smem_addr(smem + kKVOffStage + s * 2 * kTileBytes);
        const uint32_t sDO = sQ + kTileBytes;
        const uint32_t cST = bb * 128, cDPT = cST + 64;
        if (!mbar_wait(smem_addr(&bars.p_ready[bb]), ph, ab)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kHalf / 16; kk++)
          mma_ts(tmem + colDV, tmem + cST + kk * 8, mn_desc(sDO, kk, hf * kHalf), idesc_g,
                 (u > 0 || kk > 0));
        if (!mbar_wait(smem_addr(&bars.ds_ready[bb]), ph, ab)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kHalf / 16; kk++)
          mma_ts(tmem + colDK, tmem + cDPT + kk * 8, mn_desc(sQ, kk, hf * kHalf), idesc_g,
                 (u > 0 || kk > 0));
        if (hf == 1) mma_commit(smem_addr(&bars.q_empty[s]));
      }
      mma_commit(smem_addr(&bars.acc_done));
      mma_commit(smem_addr(&bars.drain));
      int no_abort = 0;
      Abort local{&no_abort, p.status};
      mbar_wait(smem_addr(&bars.drain), 0, local);
    }
  } else {
    // ------------------------------------------------------------------ per key row math
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;  // key row inside the tile
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const float sl2 = p.scale_log2;
    bool ok = true;
    for (int u = 0; u < nsteps; u++) {
      const int n = u >> 1, hf = u & 1, s = n & 1, bb = u & 1;
      const int it = it0 + n % nq;
      ok = mbar_wait(smem_addr(&bars.sdp_full[bb]), (u >> 1) & 1, ab);
      __syncwarp();
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
      const float* lse_s = reinterpret_cast<const float*>(smem + kKVOffLse + s * 512) + hf * kHalf;
      const float* d_s = reinterpret_cast<const float*>(smem + kKVOffD + s * 512) + hf * kHalf;
      const bool diag = p.causal && it == kt;
      const uint32_t tST = tmem + lane_off + bb * 128, tDPT = tST + 64;
      float pr[kHalf];
#pragma unroll
      for (int ch = 0; ch < 2; ch++) {
        uint32_t x[32];
        tmem_ld32(tST + ch * 32, x);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 32; c++) {
          const int i = ch * 32 + c;  // query row inside the half
          float v = fast_exp2(fmaf(__uint_as_float(x[c]), sl2, -lse_s[i] * kLog2e));
          if (diag && hf * kHalf + i < row) v = 0.f;
          pr[i] = v;
        }
#pragma unroll
        for (int t = 0; t < 16; t++) pk[t] = pack_bf16x2(pr[ch * 32 + 2 * t], pr[ch * 32 + 2 * t + 1]);
        tmem_st16(tST + ch * 16, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(smem_addr(&bars.p_ready[bb]));
#pragma unroll
      for (int ch = 0; ch < 2; ch++) {
        uint32_t x[32];
        tmem_ld32(tDPT + ch * 32, x);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int t = 0; t < 16; t++) {
          const int i = ch * 32 + 2 * t;
          const float d0 = pr[i] * (__uint_as_float(x[2 * t]) - d_s[i]);
          const float d1 = pr[i + 1] * (__uint_as_float(x[2 * t + 1]) - d_s[i + 1]);
          pk[t] = pack_bf16x2(d0, d1);
        }
        tmem_st16(tDPT + ch * 16, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(smem_addr(&bars.ds_ready[bb]));
    }
    if (ok) {
      ok = mbar_wait(smem_addr(&bars.acc_done), 0, ab);
      __syncwarp();
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      tc_fence_after();
      const int m = src_row(g * p.G + kt * kTile + row, sh, p.G, p.N);
      const size_t off = ((size_t)(b * p.N + m) * p.Hkv + kvh) * kD;
      __nv_bfloat16* dk = static_cast<__nv_bfloat16*>(p.dk) + off;
      __nv_bfloat16* dv = static_cast<__nv_bfloat16*>(p.dv) + off;
      const float2* cs_row = p.cs + (size_t)m * (kD / 2);
#pragma unroll
      for (int ch = 0; ch < 4; ch++) {
        uint32_t x[32];
        uint4 o[4];
        tmem_ld32(tmem + lane_off + colDK + ch * 32, x);
        tmem_wait_ld();
        unrotate_pack(x, cs_row, ch * 16, p.scale, o);
        uint4* dst = reinterpret_cast<uint4*>(dk + ch * 32);
#pragma unroll
        for (int t = 0; t < 4; t++) dst[t] = o[t];
        tmem_ld32(tmem + lane_off + colDV + ch * 32, x);
        tmem_wait_ld();
        scale_pack(x, 1.f, o);
        dst = reinterpret_cast<uint4*>(dv + ch * 32);
#pragma unroll
        for (int t = 0; t < 4; t++) dst[t] = o[t];
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ================================================================================ dQ

// smem: Q | dO | stage 0: K, V | stage 1: K, V
constexpr uint32_t kQOffQ = 0;
constexpr uint32_t kQOffDO = kTileBytes;
constexpr uint32_t kQOffStage = 2 * kTileBytes;  // + s * 2 * kTileBytes: K then V
constexpr uint32_t kQSmem = 6 * kTileBytes + 1024;

struct DqBarriers {
  uint64_t q_full;
  uint64_t kv_full[2], kv_empty[2];
  uint64_t sdp_full[2], ds_ready[2];
  uint64_t acc_done, drain;
};

__global__ void __launch_bounds__(kThreads, 1)
    tc_dq_kernel(const Params p, const __grid_constant__ CUtensorMap tm_q,
                 const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                 const __grid_constant__ CUtensorMap tm_do) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  __shared__ DqBarriers bars;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = p.G / kTile, ng = p.N / p.G, R = p.Hq / p.Hkv;
  // head-group-major: the query tiles of all query heads of one (b, kv head, group) run
  // together (they share K and V), heaviest query tiles first
  const int per_kg = T * R;
  const int inner = (int)(blockIdx.x % per_kg);
  const int bkg = (int)(blockIdx.x / per_kg);
  const int qt = T - 1 - inner / R;
  const int g = bkg % ng, bk = bkg / ng;
  const int kvh = bk % p.Hkv, b = bk / p.Hkv;
  const int h = kvh * R + inner % R;
  const bool sh = head_shifted(h, p.Hq);
  const int nkv = p.causal ? qt + 1 : T;
  const int nsteps = 2 * nkv;
  const int mq0 = src_row(g * p.G + qt * kTile, sh, p.G, p.N);

  Abort ab{&abort_flag, p.status};
  if (threadIdx.x == 0) {
    abort_flag = *reinterpret_cast<volatile unsigned*>(p.status) != 0u;
    mbar_init(smem_addr(&bars.q_full), 1);
    for (int s = 0; s < 2; s++) {
      mbar_init(smem_addr(&bars.kv_full[s]), 1);
      mbar_init(smem_addr(&bars.kv_empty[s]), 1);
      mbar_init(smem_addr(&bars.sdp_full[s]), 1);
      mbar_init(smem_addr(&bars.ds_ready[s]), 128);
    }
    mbar_init(smem_addr(&bars.acc_done), 1);
    mbar_init(smem_addr(&bars.drain), 1);
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(smem_addr(&tmem_base_sh), kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  const uint32_t colDQ = 256;
  const uint32_t sQ = smem_addr(smem + kQOffQ), sDO = smem_addr(smem + kQOffDO);
  const bool skip = abort_flag != 0;

  if (skip) {
  } else if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      const uint32_t qb = smem_addr(&bars.q_full);
      mbar_arrive_expect_tx(qb, 2 * kTileBytes);
      const int qrow = (b * p.Hq + h) * p.N + mq0;
      tma_load_2d(sQ, &tm_q, qb, 0, qrow);
      tma_load_2d(sQ + kBoxBytes, &tm_q, qb, 64, qrow);
      tma_load_3d(sDO, &tm_do, qb, 0, h, b * p.N + mq0);
      tma_load_3d(sDO + kBoxBytes, &tm_do, qb, 64, h, b * p.N + mq0);
      int issued = 0;
      for (int j = 0; j < nkv; j++) {
        const int s = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        const int mk = src_row(g * p.G + j * kTile, sh, p.G, p.N);
        if (!mbar_wait(smem_addr(&bars.kv_empty[s]), ph ^ 1, ab)) break;
        const uint32_t kb = smem_addr(&bars.kv_full[s]);
        const uint32_t sKs = smem_addr(smem + kQOffStage + s * 2 * kTileBytes);
        const uint32_t sVs = sKs + kTileBytes;
        mbar_arrive_expect_tx(kb, 2 * kTileBytes);
        const int krow = (b * p.Hkv + kvh) * p.N + mk;
        tma_load_2d(sKs, &tm_k, kb, 0, krow);
        tma_load_2d(sKs + kBoxBytes, &tm_k, kb, 64, krow);
        tma_load_3d(sVs, &tm_v, kb, 0, kvh, b * p.N + mk);
        tma_load_3d(sVs + kBoxBytes, &tm_v, kb, 64, kvh, b * p.N + mk);
        issued = j + 1;
      }
      int no_abort = 0;
      Abort local{&no_abort, p.status};
      for (int j = issued - 1; j >= 0 && j >= issued - 2; j--)
        mbar_wait(smem_addr(&bars.kv_full[j & 1]), (j >> 1) & 1, local);
      mbar_wait(qb, 0, local);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16_f32(kTile, kHalf, false, false);
      const uint32_t idesc_g = idesc_bf16_f32(kTile, kD, false, true);
      bool ok = mbar_wait(smem_addr(&bars.q_full), 0, ab);
      auto issue_scores = [&](int u) -> bool {
        const int j = u >> 1, hf = u & 1, s = j & 1;
        if (hf == 0 && !mbar_wait(smem_addr(&bars.kv_full[s]), (j >> 1) & 1, ab)) return false;
        tc_fence_after();
        const uint32_t sKs = smem_addr(smem + kQOffStage + s * 2 * kTileBytes);
        const uint32_t sVs = sKs + kTileBytes;
        const uint32_t cS = (u & 1) * 128, cDP = cS + 64;
#pragma unroll
        for (int kk = 0; kk < kD / 16; kk++)
          mma_ss(tmem + cS, kmajor_desc(sQ, kk), kmajor_desc(sKs, kk, hf * kHalf), idesc_s, kk > 0);
#pragma unroll
        for (int kk = 0; kk < kD / 16; kk++)
          mma_ss(tmem + cDP, kmajor_desc(sDO, kk), kmajor_desc(sVs, kk, hf * kHalf), idesc_s,
                 kk > 0);
        mma_commit(smem_addr(&bars.sdp_full[u & 1]));
        return true;
      };
      tc_fence_after();
      if (ok && nsteps > 0) ok = issue_scores(0);
      for (int u = 0; ok && u < nsteps; u++) {
        if (u + 1 < nsteps && !issue_scores(u + 1)) break;
        const int j = u >> 1, hf = u & 1, s = j & 1, bb = u & 1;
        const uint32_t sKs = smem_addr(smem + kQOffStage + s * 2 * kTileBytes);
        if (!mbar_wait(smem_addr(&bars.ds_ready[bb]), (u >> 1) & 1, ab)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kHalf / 16; kk++)
          mma_ts(tmem + colDQ, tmem + bb * 128 + kk * 8, mn_desc(sKs, kk, hf * kHalf), idesc_g,
                 (u > 0 || kk > 0));
        if (hf == 1) mma_commit(smem_addr(&bars.kv_empty[s]));
      }
      mma_commit(smem_addr(&bars.acc_done));
      mma_commit(smem_addr(&bars.drain));
      int no_abort = 0;
      Abort local{&no_abort, p.status};
      mbar_wait(smem_addr(&bars.drain), 0, local);
    }
  } else {
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;  // query row inside the tile
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const int m = src_row(g * p.G + qt * kTile + row, sh, p.G, p.N);
    const size_t lrow = ((size_t)b * p.Hq + h) * p.N + m;
    const float nlse2 = -p.lse[lrow] * kLog2e;
    const float Dm = p.Dsum[lrow];
    const float sl2 = p.scale_log2;
    bool ok = true;
    for (int u = 0; u < nsteps; u++) {
      const int j = u >> 1, hf = u & 1, bb = u & 1;
      ok = mbar_wait(smem_addr(&bars.sdp_full[bb]), (u >> 1) & 1, ab);
      __syncwarp();
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
      const bool diag = p.causal && j == qt;
      const uint32_t tS = tmem + lane_off + bb * 128, tDP = tS + 64;
#pragma unroll
      for (int ch = 0; ch < 2; ch++) {
        uint32_t xs[32], xd[32];
        tmem_ld32(tS + ch * 32, xs);
        tmem_ld32(tDP + ch * 32, xd);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int t = 0; t < 16; t++) {
          const int c0 = hf * kHalf + ch * 32 + 2 * t;  // key column inside its tile
          float p0 = fast_exp2(fmaf(__uint_as_float(xs[2 * t]), sl2, nlse2));
          float p1 = fast_exp2(fmaf(__uint_as_float(xs[2 * t + 1]), sl2, nlse2));
          if (diag && c0 > row) p0 = 0.f;
          if (diag && c0 + 1 > row) p1 = 0.f;
          pk[t] = pack_bf16x2(p0 * (__uint_as_float(xd[2 * t]) - Dm),
                              p1 * (__uint_as_float(xd[2 * t + 1]) - Dm));
        }
        tmem_st16(tS + ch * 16, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(smem_addr(&bars.ds_ready[bb]));
    }
    if (ok) {
      ok = mbar_wait(smem_addr(&bars.acc_done), 0, ab);
      __syncwarp();
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      tc_fence_after();
      __nv_bfloat16* dq = static_cast<__nv_bfloat16*>(p.dq) + ((size_t)(b * p.N + m) * p.Hq + h) * kD;
      const float2* cs_row = p.cs + (size_t)m * (kD / 2);
#pragma unroll
      for (int ch = 0; ch < 4; ch++) {
        uint32_t x[32];
        uint4 o[4];
        tmem_ld32(tmem + lane_off + colDQ + ch * 32, x);
        tmem_wait_ld();
        unrotate_pack(x, cs_row, ch * 16, p.scale, o);
        uint4* dst = reinterpret_cast<uint4*>(dq + ch * 32);
#pragma unroll
        for (int t = 0; t < 4; t++) dst[t] = o[t];
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

cudaError_t make_bwd_maps(const Params& p, CUtensorMap* tq, CUtensorMap* tk, CUtensorMap* tv,
                          CUtensorMap* tdo) {
  cudaError_t e;
  if ((e = make_tmap_bf16_2d(tq, p.qr, kD, (uint64_t)p.B * p.Hq * p.N, kD * 2, 64, kTile)))
    return e;
  if ((e = make_tmap_bf16_2d(tk, p.kr, kD, (uint64_t)p.B * p.Hkv * p.N, kD * 2, 64, kTile)))
    return e;
  if ((e = make_tmap_bf16_3d(tv, p.v, kD, p.Hkv, (uint64_t)p.B * p.N, kD * 2,
                             (uint64_t)p.Hkv * kD * 2, 64, kTile)))
    return e;
  return make_tmap_bf16_3d(tdo, p.dout, kD, p.Hq, (uint64_t)p.B * p.N, kD * 2,
                           (uint64_t)p.Hq * kD * 2, 64, kTile);
}

}  // namespace

cudaError_t launch_tc_bwd_dkdv(const Params& p, cudaStream_t st) {
  CUtensorMap tq, tk, tv, tdo;
  cudaError_t e = make_bwd_maps(p, &tq, &tk, &tv, &tdo);
  if (e) return e;
  if ((e = cudaFuncSetAttribute(tc_dkdv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)kKVSmem)))
    return e;
  const long tiles = (long)p.B * p.Hkv * (p.N / p.G) * (p.G / kTile);
  tc_dkdv_kernel<<<dim3((unsigned)tiles), dim3(kThreads), kKVSmem, st>>>(p, tq, tk, tv, tdo);
  return cudaGetLastError();
}

cudaError_t launch_tc_bwd_dq(const Params& p, cudaStream_t st) {
  CUtensorMap tq, tk, tv, tdo;
  cudaError_t e = make_bwd_maps(p, &tq, &tk, &tv, &tdo);
  if (e) return e;
  if ((e = cudaFuncSetAttribute(tc_dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)kQSmem)))
    return e;
  const long tiles = (long)p.B * p.Hq * (p.N / p.G) * (p.G / kTile);
  tc_dq_kernel<<<dim3((unsigned)tiles), dim3(kThreads), kQSmem, st>>>(p, tq, tk, tv, tdo);
  return cudaGetLastError();
}

}  // namespace s2
