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
// Keeping the tensor cores busy. Per pair of 128-row tiles both passes run three or four
// 128 x 128 x 128 MMAs and one round of per-row math that depends on two of them. The
// math warps first load the score tile (S, or S^T) into registers and release it at once,
// so the next pair's score MMA can run while they compute; they write the bf16 operands
// of the gradient MMAs (P^T and dS^T, or dS) over the dP tile after loading it. The MMA
// queue therefore always holds work: gradient MMAs of pair n, dP of pair n+1, scores of
// pair n+2 (issued last, so it never delays the MMAs the next math phase waits for).
// Eight math warps share the rows (two per TMEM lane quarter, 64 columns each).
//
// dK/dV pass: one CTA per 128-row key tile (b, kv head, group, kt). For every query head of
// the kv head and every query tile it >= kt (causal):
//     S^T  = K Q^T       (SS MMA)             TMEM [0,128)     thread = key row = lane
//     dP^T = V dO^T      (SS MMA)             TMEM [128,256)
//     P^T  = exp2(S^T log2(e)/sqrt(d) - LSE_i log2(e)), dS^T = P^T (dP^T - D_i), both bf16,
//            written over dP^T: per 32 query rows, P^T in 16 columns and dS^T in the next 16
//     dV  += P^T dO      (TS MMA)             TMEM [256,384)
//     dK  += dS^T Q      (TS MMA)             TMEM [384,512)
//   The GQA sum over query heads happens in the TMEM accumulators (no atomics).
//   Epilogue: dk = R^T (dK / sqrt(d)), dv = dV, bf16, at the key tokens' original rows.
// dQ pass: persistent CTAs take 128-row query tiles (b, head, group, qt) from a work counter.
// For every key tile j <= qt:
//   S = Q K^T (TMEM [0,128)), dP = dO V^T into one of two buffers ([128,256), [256,384)),
//   dS = P (dP - D) bf16 over that dP (the first 32 of each math warp's 64 columns),
//   dQ += dS K (TS MMA, [384,512)). Three MMA issuers (warp 1: S, warp 2: dP, warp 3: dQ),
//   see the kernel. Epilogue: dq = R^T (dQ / sqrt(d)), bf16, at the query tokens' original rows.
// Work is numbered a few (b, kv head, group) units at a time, heaviest items first within
// them (chunked_lpt), so the CTAs running together share the tiles they stream (L2 reuse)
// and the last wave is light. Roles: warp 0 TMA producer, warp 1 MMA issuer and TMEM owner,
// (dQ pass: warps 1..3 MMA issuers), warps 4..11 the per-row math, whose elementwise work
// runs on packed fp32 pairs (f32x2). Every wait is bounded (see sm100.cuh).
#include "common.cuh"
#include "fastmath.cuh"
#include "sm100.cuh"
#include "tc_kernels.h"
#include "tma_host.h"

namespace s2 {
namespace {

using namespace sm100;

constexpr int kD = 128;
constexpr int kTile = 128;
constexpr uint32_t kTileBytes = kTile * kD * 2;
constexpr uint32_t kBoxBytes = kTileBytes / 2;     // one 128-row x 64-column TMA box
constexpr int kThreads = 384;
constexpr int kMathThreads = 256;
constexpr uint32_t kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Columns c, c+1 of a thread's 64 loaded TMEM values, as a packed fp32 pair.
__device__ __forceinline__ uint64_t score_pair(const uint32_t (&x0)[32], const uint32_t (&x1)[32],
                                               int c) {
  return c < 32 ? f2pack(__uint_as_float(x0[c]), __uint_as_float(x0[c + 1]))
                : f2pack(__uint_as_float(x1[c - 32]), __uint_as_float(x1[c - 31]));
}

// K-major operand (128 rows x 128 bf16 in two 64-column SW128 boxes), k-step kk.
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t tile_saddr, int kk) {
  return smem_desc_sw128(tile_saddr + (kk >> 2) * kBoxBytes + (kk & 3) * 32, 16, 1024);
}

// Tile rows as an MN-major B operand (K = rows, N = d): k-step kk covers rows 16kk..16kk+15.
__device__ __forceinline__ uint64_t mn_desc(uint32_t tile_saddr, int kk) {
  return smem_desc_sw128(tile_saddr + kk * 2048, kBoxBytes, 1024);
}

// The same descriptors' offsets (in 16-byte units) from the tile's k-step 0 descriptor.
__device__ __forceinline__ uint64_t kmajor_koff(int kk) {
  return (uint64_t)(((kk >> 2) * kBoxBytes + (kk & 3) * 32) >> 4);
}
__device__ __forceinline__ uint64_t mn_koff(int kk) { return (uint64_t)((kk * 2048) >> 4); }
constexpr uint32_t kTileDesc = kTileBytes >> 4;  // one tile, in descriptor address units

// Keeps a value in a register as an opaque quantity, so that the descriptors derived from it
// per stage and k-step are formed by one add where they are used instead of being hoisted
// out of the loops (and spilled).
__device__ __forceinline__ uint64_t opaque64(uint64_t v) {
  uint64_t r;
  asm volatile("mov.b64 %0, %1;" : "=l"(r) : "l"(v));
  return r;
}

// The dQ pass: bit t set sends the exponentials of column pair t (columns 2t, 2t+1 of a
// math warp's 64) to the packed FMA-pipe polynomial (fastmath.cuh), else to the MUFU unit;
// off the diagonal tiles only (no -inf scores there; the polynomial clamps its argument at
// -125). On a B200, 32k workload, 1/8, 1/4 and 3/8 of them there gave 2.65-2.68 /
// 2.67-2.70 / 2.64-2.68 ms against 2.63-2.66 ms with none (within run-to-run noise): the
// pass is not bound by the MUFU, so the default is none.
#ifndef S2_DQ_POLY_MASK
#define S2_DQ_POLY_MASK 0x0u
#endif
constexpr unsigned kDqPolyMask = S2_DQ_POLY_MASK;
// The dK/dV pass: bit t set sends the exponentials of column pair t (columns 2t, 2t+1 of a
// math warp's 64) to the packed FMA-pipe polynomial, off the diagonal tiles. On a B200, 32k
// workload, 1/8, 1/4 and 1/2 of them there gave 3.52 / 3.62 / 3.68 ms against 3.59-3.68 ms
// with none (within run-to-run noise): the pass is not bound by the MUFU, so the default
// is none.
#ifndef S2_DKDV_POLY_MASK
#define S2_DKDV_POLY_MASK 0x0u
#endif
constexpr unsigned kDkdvPolyMask = S2_DKDV_POLY_MASK;

// Causal mask of a diagonal tile, applied to a thread's 64 raw scores (columns c = 0..63 of
// its half) before the exponential: the score becomes -inf, so its probability is exactly 0.
// upper = 0 masks the columns c < lim, upper = 1 the columns c > lim. Called only on the
// diagonal tile (a warp-uniform branch), so the other tiles pay nothing for the mask.
__device__ __forceinline__ void mask_scores(uint32_t (&x0)[32], uint32_t (&x1)[32], int lim,
                                            int upper) {
  const uint32_t ninf = 0xff800000u;
#pragma unroll
  for (int c = 0; c < 32; c++) {
    if (upper ? c > lim : c < lim) x0[c] = ninf;
    if (upper ? c + 32 > lim : c + 32 < lim) x1[c] = ninf;
  }
}

// Makes the 64 values count as used here: the exponentials of the probabilities are then
// computed before the wait that follows (while the tensor cores work) instead of being
// scheduled after it, where they would lengthen the critical path of the next MMA.
__device__ __forceinline__ void pin_regs(float (&x)[64]) {
#pragma unroll
  for (int c = 0; c < 64; c++) asm volatile("" : "+f"(x[c]));
}

// TMEM column of the bf16 A operand for k-step kk (16 K rows = 8 packed columns) in the dQ
// pass. Each math warp owns 64 K rows (columns c0 = 0 or 64 of the tile) and writes dS
// chunk by chunk (32 K rows each) into the first 16 of each 32 fp32 columns it has just
// read: region + c0 + 16 * chunk .. + 16.
__device__ __forceinline__ uint32_t packed_col(uint32_t region, int kk) {
  return region + (kk >> 2) * 64 + ((kk >> 1) & 1) * 16 + (kk & 1) * 8;
}

// ================================================================================ dK / dV

// smem: K | V | Q stages 0..2 (each a 32 KB tile followed by its 4 KB row-term block) | dO |
// the two constant row-term operands (4 KB each). After the last pair the K, V region holds
// the (cos, sin) rows of the key tile and Q stages 0, 1 the bf16 dK, dV tiles on their way out.
constexpr int kQStages = 3;
constexpr uint32_t kTermBytes = kTile * 16 * 2;              // 128 rows x 16 bf16, SW32
constexpr uint32_t kQStageBytes = kTileBytes + kTermBytes;
constexpr uint32_t kKVOffK = 0;
constexpr uint32_t kKVOffV = kTileBytes;
constexpr uint32_t kKVOffQ = 2 * kTileBytes;
constexpr uint32_t kKVOffDO = kKVOffQ + kQStages * kQStageBytes;
constexpr uint32_t kKVOffKTerm = kKVOffDO + kTileBytes;
constexpr uint32_t kKVOffVTerm = kKVOffKTerm + kTermBytes;
constexpr uint32_t kKVSmem = kKVOffVTerm + kTermBytes + 1024;
#ifndef S2_DKDV_PREFETCH_AHEAD
#define S2_DKDV_PREFETCH_AHEAD 2
#endif
constexpr int kPrefetchAhead = S2_DKDV_PREFETCH_AHEAD;  // pairs between L2 prefetch and use
constexpr uint32_t kCsBoxBytes = kTile * 32 * 4;         // 128 rows x 32 floats

struct DkdvBarriers {
  uint64_t kv_full, cs_full;
  uint64_t q_full[kQStages], q_empty[kQStages];
  uint64_t do_full, do_empty;
  uint64_t st_full, p_ready, dpt_full, ds_ready;
  uint64_t kv_free, acc_done, drain;
};

// One row of the constant operand of the row-term k-step: bf16 ones at the given element
// positions of the 16, the same in both 16-byte halves (so the row reads the same under the
// 32-byte swizzle whichever half comes first; the row-term rows are zero in elements 8..15).
__device__ __forceinline__ uint4 term_row_half(int first, int count) {
  uint32_t w[4] = {0u, 0u, 0u, 0u};
  for (int e = first; e < first + count; e++) w[e >> 1] |= 0x3F80u << ((e & 1) * 16);
  return make_uint4(w[0], w[1], w[2], w[3]);
}

__global__ void __launch_bounds__(kThreads, 1)
    tc_dkdv_kernel(const Params p, const __grid_constant__ CUtensorMap tm_q,
                   const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                   const __grid_constant__ CUtensorMap tm_do,
                   const __grid_constant__ CUtensorMap tm_terms,
                   const __grid_constant__ CUtensorMap tm_cs,
                   const __grid_constant__ CUtensorMap tm_dk,
                   const __grid_constant__ CUtensorMap tm_dv) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  __shared__ DkdvBarriers bars;
  __shared__ uint32_t tmem_base_sh;
  __shared__ AbortState abort_state;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = p.G / kTile, ng = p.N / p.G, R = p.Hq / p.Hkv;
  // the key tiles of a few (b, kv head, group) units run together (they stream the same Q
  // and dO through L2), heaviest first: key tile kt sees T - kt query tiles when causal
  int kt, bkg;
  chunked_lpt((int)blockIdx.x, p.B * p.Hkv * ng, T, bkg, kt);
  const int g = bkg % ng, bk = bkg / ng;
  const int kvh = bk % p.Hkv, b = bk / p.Hkv;
  const bool sh = kv_head_shifted(kvh, p);
  const int it0 = p.causal ? kt : 0;
  const int nq = T - it0;      // query tiles per query head
  const int np = R * nq;       // (query head, query tile) pairs
  const int mk0 = src_row(g * p.G + kt * kTile, sh, p.G, p.N);

  // the constant operands of the row-term k-step: ones against -LSE*sqrt(d) (elements
  // 0..2) for S^T, against -D (elements 3, 4) for dP^T
  {
    const uint4 kt_half = term_row_half(0, 3), vt_half = term_row_half(3, 2);
    uint4* kterm = reinterpret_cast<uint4*>(smem + kKVOffKTerm);
    uint4* vterm = reinterpret_cast<uint4*>(smem + kKVOffVTerm);
    for (int i = threadIdx.x; i < (int)(kTermBytes / 16); i += kThreads) {
      kterm[i] = kt_half;
      vterm[i] = vt_half;
    }
    fence_proxy_async_shared();
  }
  const Abort ab{smem_addr(&abort_state)};
  if (threadIdx.x == 0) {
    abort_state_init(abort_state, p.status, p.wait_limit_ns,
                     *reinterpret_cast<volatile unsigned*>(p.status) != 0u);
    mbar_init(smem_addr(&bars.kv_full), 1);
    mbar_init(smem_addr(&bars.cs_full), 1);
    for (int s = 0; s < kQStages; s++) {
      mbar_init(smem_addr(&bars.q_full[s]), 1);
      mbar_init(smem_addr(&bars.q_empty[s]), 1);
    }
    mbar_init(smem_addr(&bars.do_full), 1);
    mbar_init(smem_addr(&bars.do_empty), 1);
    mbar_init(smem_addr(&bars.st_full), 1);
    mbar_init(smem_addr(&bars.p_ready), kMathThreads);
    mbar_init(smem_addr(&bars.dpt_full), 1);
    mbar_init(smem_addr(&bars.ds_ready), kMathThreads);
    mbar_init(smem_addr(&bars.kv_free), 1);
    mbar_init(smem_addr(&bars.acc_done), 1);
    mbar_init(smem_addr(&bars.drain), 1);
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(smem_addr(&tmem_base_sh), kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  const uint32_t colST = 0, colDPT = 128, colDV = 256, colDK = 384;
  const uint32_t sK = smem_addr(smem + kKVOffK), sV = smem_addr(smem + kKVOffV);
  const uint32_t sDO = smem_addr(smem + kKVOffDO);
  const bool skip = abort_state.flag != 0;

  // Pairs run query tile it0 .. T-1 of query head kvh*R, then of the next head, and so on.
  // Each role walks them with a cursor (no division by nq: an integer division uses the
  // MUFU reciprocal, which the math warps' exponentials keep busy).
  struct PairCursor {
    int h, iq;
  };
  auto pair_first = [&]() { return PairCursor{kvh * R, it0}; };
  auto pair_next = [&](PairCursor& c) {
    if (++c.iq == T) {
      c.iq = it0;
      ++c.h;
    }
  };
  auto pair_row0 = [&](const PairCursor& c) {
    return src_row(g * p.G + c.iq * kTile, sh, p.G, p.N);
  };

  if (skip) {
  } else if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer: K, V, Q
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      tma_prefetch_desc(&tm_terms);
      tma_prefetch_desc(&tm_cs);
      const uint32_t kvb = smem_addr(&bars.kv_full);
      mbar_arrive_expect_tx(kvb, 2 * kTileBytes);
      const int krow = (b * p.Hkv + kvh) * p.N + mk0;
      tma_load_2d(sK, &tm_k, kvb, 0, krow);
      tma_load_2d(sK + kBoxBytes, &tm_k, kvb, 64, krow);
      tma_load_3d(sV, &tm_v, kvb, 0, kvh, b * p.N + mk0);
      tma_load_3d(sV + kBoxBytes, &tm_v, kvb, 64, kvh, b * p.N + mk0);
      {
        // the K, V tiles of the CTA that will most likely follow this one on an SM (one
        // SM's worth of CTAs later) into L2, so that its first loads hit there
        unsigned nsm;
        asm("mov.u32 %0, %%nsmid;" : "=r"(nsm));
        const int nx = (int)blockIdx.x + (int)nsm;
        if (nx < (int)gridDim.x) {
          int kt2, bkg2;
          chunked_lpt(nx, p.B * p.Hkv * ng, T, bkg2, kt2);
          const int g2 = bkg2 % ng, bk2 = bkg2 / ng;
          const int kvh2 = bk2 % p.Hkv, b2 = bk2 / p.Hkv;
          const int mk2 = src_row(g2 * p.G + kt2 * kTile, kv_head_shifted(kvh2, p), p.G, p.N);
          const int krow2 = (b2 * p.Hkv + kvh2) * p.N + mk2;
          tma_prefetch_l2_2d(&tm_k, 0, krow2);
          tma_prefetch_l2_2d(&tm_k, 64, krow2);
          tma_prefetch_l2_3d(&tm_v, 0, kvh2, b2 * p.N + mk2);
          tma_prefetch_l2_3d(&tm_v, 64, kvh2, b2 * p.N + mk2);
        }
      }
      int nq_issued = 0;
      PairCursor pc = pair_first(), pf = pair_first();
      for (int t = 0; t < kPrefetchAhead; t++) pair_next(pf);
      for (int n = 0; n < np; n++, pair_next(pc), pair_next(pf)) {
        const int h = pc.h, mq0 = pair_row0(pc);
        const int sq = n % kQStages;
        // the Q and dO tiles of pair n + kPrefetchAhead into L2 before this thread blocks on
        // a free ring stage: their loads into shared memory then hit in L2
        if (n + kPrefetchAhead < np) {
          const int mqp = pair_row0(pf);
          const int qrowp = (b * p.Hq + pf.h) * p.N + mqp;
          tma_prefetch_l2_2d(&tm_q, 0, qrowp);
          tma_prefetch_l2_2d(&tm_q, 64, qrowp);
          tma_prefetch_l2_3d(&tm_do, 0, pf.h, b * p.N + mqp);
          tma_prefetch_l2_3d(&tm_do, 64, pf.h, b * p.N + mqp);
        }
        if (!mbar_wait(smem_addr(&bars.q_empty[sq]), ((n / kQStages) & 1) ^ 1, ab)) break;
        const uint32_t qb = smem_addr(&bars.q_full[sq]);
        const uint32_t sQ = smem_addr(smem + kKVOffQ + sq * kQStageBytes);
        mbar_arrive_expect_tx(qb, kQStageBytes);
        const int qrow = (b * p.Hq + h) * p.N + mq0;
        tma_load_2d(sQ, &tm_q, qb, 0, qrow);
        tma_load_2d(sQ + kBoxBytes, &tm_q, qb, 64, qrow);
        tma_load_2d(sQ + kTileBytes, &tm_terms, qb, 0, qrow);
        nq_issued = n + 1;
      }
      // once the last MMA that reads K and V has completed, the (cos, sin) rows of the key
      // tile (the epilogue's inverse rotation) take their place
      bool cs_issued = false;
      if (nq_issued == np && mbar_wait(smem_addr(&bars.kv_free), 0, ab)) {
        const uint32_t cb = smem_addr(&bars.cs_full);
        mbar_arrive_expect_tx(cb, 4 * kCsBoxBytes);
        for (int x = 0; x < 4; x++) tma_load_2d(sK + x * kCsBoxBytes, &tm_cs, cb, 32 * x, mk0);
        cs_issued = true;
      }
      for (int n = nq_issued - 1; n >= 0 && n >= nq_issued - kQStages; n--)
        mbar_wait_drain(smem_addr(&bars.q_full[n % kQStages]), (n / kQStages) & 1, p.status,
                        p.wait_limit_ns);
      mbar_wait_drain(kvb, 0, p.status, p.wait_limit_ns);
      if (cs_issued) mbar_wait_drain(smem_addr(&bars.cs_full), 0, p.status, p.wait_limit_ns);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------------ TMA producer: dO
    if (lane == 0) {
      int ndo_issued = 0;
      PairCursor pc = pair_first();
      for (int n = 0; n < np; n++, pair_next(pc)) {
        if (!mbar_wait(smem_addr(&bars.do_empty), (n & 1) ^ 1, ab)) break;
        const uint32_t db = smem_addr(&bars.do_full);
        const int mq0 = pair_row0(pc);
        mbar_arrive_expect_tx(db, kTileBytes);
        tma_load_3d(sDO, &tm_do, db, 0, pc.h, b * p.N + mq0);
        tma_load_3d(sDO + kBoxBytes, &tm_do, db, 64, pc.h, b * p.N + mq0);
        ndo_issued = n + 1;
      }
      if (ndo_issued > 0)
        mbar_wait_drain(smem_addr(&bars.do_full), (ndo_issued - 1) & 1, p.status,
                        p.wait_limit_ns);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    // The whole warp runs the issue loop (warp-uniform control flow and descriptors); one
    // elected lane issues each MMA and commit.
    {
      const uint32_t idesc_s = idesc_bf16_f32(kTile, kTile, false, false);
      const uint32_t idesc_g = idesc_bf16_f32(kTile, kD, false, true);
      const uint64_t dKT = smem_desc_sw32(smem_addr(smem + kKVOffKTerm));
      const uint64_t dVT = smem_desc_sw32(smem_addr(smem + kKVOffVTerm));
      auto stage_q = [&](int n) { return smem_addr(smem + kKVOffQ + (n % kQStages) * kQStageBytes); };
      // S^T(n) - LSE*sqrt(d) = K Q_n^T + 1 (row terms)^T: eight k-steps and the row-term step
      auto issue_st = [&](int n) -> bool {
        const int sq = n % kQStages;
        if (!__all_sync(0xffffffffu, mbar_wait(smem_addr(&bars.q_full[sq]), (n / kQStages) & 1, ab)))
          return false;
        tc_fence_after();
        const uint32_t sQ = stage_q(n);
#pragma unroll
        for (int kk = 0; kk < kD / 16; kk++)
          mma_ss_elect(tmem + colST, kmajor_desc(sK, kk), kmajor_desc(sQ, kk), idesc_s, kk > 0);
        mma_ss_elect(tmem + colST, dKT, smem_desc_sw32(sQ + kTileBytes), idesc_s, 1u);
        // failure-path self-test: CTA 0 (key tile 0, at least two pairs) withholds the
        // arrival of S^T(1), so that the math warps and then this thread wait in vain
        if (!(p.inject == kInjectDkdv && blockIdx.x == 0 && n == 1))
          mma_commit_elect(smem_addr(&bars.st_full));
        return true;
      };
      // dP^T(n) - D = V dO_n^T + 1 (row terms)^T (the row terms sit in Q stage n)
      auto issue_dpt = [&](int n) -> bool {
        if (!__all_sync(0xffffffffu, mbar_wait(smem_addr(&bars.do_full), n & 1, ab))) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kD / 16; kk++)
          mma_ss_elect(tmem + colDPT, kmajor_desc(sV, kk), kmajor_desc(sDO, kk), idesc_s, kk > 0);
        mma_ss_elect(tmem + colDPT, dVT, smem_desc_sw32(stage_q(n) + kTileBytes), idesc_s, 1u);
        mma_commit_elect(smem_addr(&bars.dpt_full));
        return true;
      };
      // Per pair n: dV(n) once the math warps have written P^T(n) over S^T(n), then S^T(n+1)
      // over it (the MMAs run in issue order); dK(n) once they have written dS^T(n) over
      // dP^T(n), then dP^T(n+1) over it. The math warps' exponentials of pair n+1 then run
      // while dK(n) and dP^T(n+1) occupy the tensor cores.
      bool ok = __all_sync(0xffffffffu, mbar_wait(smem_addr(&bars.kv_full), 0, ab));
      tc_fence_after();
      if (ok && np > 0) ok = issue_st(0) && issue_dpt(0);
      if (ok && np == 1) mma_commit_elect(smem_addr(&bars.kv_free));
      for (int n = 0; ok && n < np; n++) {
        const uint32_t ph = n & 1;
        if (!__all_sync(0xffffffffu, mbar_wait(smem_addr(&bars.p_ready), ph, ab))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kTile / 16; kk++)
          mma_ts_elect(tmem + colDV, tmem + colST + (kk >> 2) * 64 + (kk & 3) * 8, mn_desc(sDO, kk),
                 idesc_g, (n > 0 || kk > 0));
        mma_commit_elect(smem_addr(&bars.do_empty));
        if (n + 1 < np && !issue_st(n + 1)) break;
        if (!__all_sync(0xffffffffu, mbar_wait(smem_addr(&bars.ds_ready), ph, ab))) break;
        tc_fence_after();
        const uint32_t sQ = stage_q(n);
#pragma unroll
        for (int kk = 0; kk < kTile / 16; kk++)
          mma_ts_elect(tmem + colDK, tmem + colDPT + (kk >> 2) * 64 + (kk & 3) * 8, mn_desc(sQ, kk),
                 idesc_g, (n > 0 || kk > 0));
        mma_commit_elect(smem_addr(&bars.q_empty[n % kQStages]));
        if (n + 1 < np) {
          if (!issue_dpt(n + 1)) break;
          if (n + 2 == np) mma_commit_elect(smem_addr(&bars.kv_free));  // the last reader of K, V
        }
      }
      mma_commit_elect(smem_addr(&bars.acc_done));
      mma_commit_elect(smem_addr(&bars.drain));
      mbar_wait_drain(smem_addr(&bars.drain), 0, p.status, p.wait_limit_ns);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------------ per key row math
    const int quarter = warp & 3;
    const int c0 = ((warp - 4) >> 2) * 64;  // this warp's 64 query columns of the tile
    const int row = quarter * 32 + lane;    // key row inside the tile
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tST = tmem + lane_off + colST + c0;
    const uint32_t tDPT = tmem + lane_off + colDPT + c0;
    const uint64_t sl2x2 = f2pack(p.scale_log2, p.scale_log2);
    PairCursor cur = pair_first();
    bool ok = true;
    for (int n = 0; n < np; n++) {
      const bool diag = p.causal && cur.iq == kt;
      pair_next(cur);
      ok = mbar_wait(smem_addr(&bars.st_full), n & 1, ab);
      __syncwarp();
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
      // P^T = exp2((S^T - LSE sqrt(d)) log2(e) / sqrt(d)); the row terms came with the MMA
      float pr[64];
      {
        uint32_t x0[32], x1[32];
        tmem_ld32(tST, x0);
        tmem_ld32(tST + 32, x1);
        tmem_wait_ld();
        if (diag) {
          mask_scores(x0, x1, row - c0, 0);  // query row c0+c before key row: P = 0
#pragma unroll
          for (int c = 0; c < 64; c += 2) {
            float a0, a1;
            f2unpack(fmul2(score_pair(x0, x1, c), sl2x2), a0, a1);
            pr[c] = fast_exp2(a0);
            pr[c + 1] = fast_exp2(a1);
          }
        } else {
#pragma unroll
          for (int c = 0; c < 64; c += 2) {
            const uint64_t a = fmul2(score_pair(x0, x1, c), sl2x2);
            if ((kDkdvPolyMask >> (c >> 1)) & 1u) {
              f2unpack(exp2_poly2(a), pr[c], pr[c + 1]);
            } else {
              float a0, a1;
              f2unpack(a, a0, a1);
              pr[c] = fast_exp2(a0);
              pr[c + 1] = fast_exp2(a1);
            }
          }
        }
        uint32_t pp[32];
#pragma unroll
        for (int t = 0; t < 32; t++) pp[t] = pack_bf16x2(pr[2 * t], pr[2 * t + 1]);
        tmem_st32(tST, pp);  // P^T of these 64 query rows over their scores, bf16 pairs
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(smem_addr(&bars.p_ready));
      ok = mbar_wait(smem_addr(&bars.dpt_full), n & 1, ab);
      __syncwarp();
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
      // dS^T = P^T (dP^T - D); the row terms came with the MMA
      {
        uint32_t x0[32], x1[32];
        tmem_ld32(tDPT, x0);
        tmem_ld32(tDPT + 32, x1);
        tmem_wait_ld();
        uint32_t pd[32];
#pragma unroll
        for (int t = 0; t < 32; t++) {
          float s0, s1;
          f2unpack(fmul2(f2pack(pr[2 * t], pr[2 * t + 1]), score_pair(x0, x1, 2 * t)), s0, s1);
          pd[t] = pack_bf16x2(s0, s1);
        }
        tmem_st32(tDPT, pd);  // dS^T over dP^T
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(smem_addr(&bars.ds_ready));
    }
    // Epilogue, taken by all eight math warps together or by none (every wait above is
    // bounded, so each warp gets here): dk = R^T (dK / sqrt(d)) and dv = dV as bf16 tiles in
    // shared memory (Q stages 0 and 1, 128-byte swizzle), then two TMA stores each.
    if (ok) {
      ok = mbar_wait(smem_addr(&bars.acc_done), 0, ab);
      __syncwarp();
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      ok = mbar_wait(smem_addr(&bars.cs_full), 0, ab);
      __syncwarp();
      ok = __all_sync(0xffffffffu, ok);
    }
    if (named_bar_and(1, kMathThreads, ok)) {
      tc_fence_after();
      const int sw = row & 7;
      uint8_t* const stage_dk = smem + kKVOffQ + (c0 >> 6) * kBoxBytes + row * 128;
      uint8_t* const stage_dv = smem + kKVOffQ + kQStageBytes + (c0 >> 6) * kBoxBytes + row * 128;
#pragma unroll
      for (int ch = 0; ch < 2; ch++) {
        // (cos, sin) of this row's channel pairs c0/2 + 16ch .. +15: box c0/32 + ch of the
        // table rows, 16-byte chunk j at j ^ (row & 7)
        const uint8_t* cs_row = smem + ((c0 >> 5) + ch) * kCsBoxBytes + row * 128;
        uint32_t x[32];
        tmem_ld32(tmem + lane_off + colDK + c0 + ch * 32, x);
        tmem_wait_ld();
        uint32_t w[16];
#pragma unroll
        for (int j = 0; j < 8; j++) {
          const float4 cs = *reinterpret_cast<const float4*>(cs_row + ((j ^ sw) << 4));
#pragma unroll
          for (int e = 0; e < 2; e++) {
            const int t = 2 * j + e;
            const float c = e ? cs.z : cs.x, s = e ? cs.w : cs.y;
            const float x0 = __uint_as_float(x[2 * t]) * p.scale;
            const float x1 = __uint_as_float(x[2 * t + 1]) * p.scale;
            w[t] = pack_bf16x2(fmaf(x0, c, x1 * s), fmaf(-x0, s, x1 * c));
          }
        }
#pragma unroll
        for (int u = 0; u < 4; u++)
          *reinterpret_cast<uint4*>(stage_dk + (((4 * ch + u) ^ sw) << 4)) =
              make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
        tmem_ld32(tmem + lane_off + colDV + c0 + ch * 32, x);
        tmem_wait_ld();
#pragma unroll
        for (int t = 0; t < 16; t++)
          w[t] = pack_bf16x2(__uint_as_float(x[2 * t]), __uint_as_float(x[2 * t + 1]));
#pragma unroll
        for (int u = 0; u < 4; u++)
          *reinterpret_cast<uint4*>(stage_dv + (((4 * ch + u) ^ sw) << 4)) =
              make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
      }
      fence_proxy_async_shared();
      named_bar_sync(1, kMathThreads);
      if (warp == 4 && lane == 0) {
        const uint32_t sdk = smem_addr(smem + kKVOffQ);
        const uint32_t sdv = smem_addr(smem + kKVOffQ + kQStageBytes);
        tma_store_3d(&tm_dk, sdk, 0, kvh, b * p.N + mk0);
        tma_store_3d(&tm_dk, sdk + kBoxBytes, 64, kvh, b * p.N + mk0);
        tma_store_3d(&tm_dv, sdv, 0, kvh, b * p.N + mk0);
        tma_store_3d(&tm_dv, sdv + kBoxBytes, 64, kvh, b * p.N + mk0);
        bulk_commit_group();
        bulk_wait_group_read0();  // shared memory may be released once the stores read it
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

// smem: Q | dO | K stages 0..2 | V stages 0..1
constexpr int kKStages = 3, kVStages = 2;
constexpr uint32_t kQOffQ = 0;
constexpr uint32_t kQOffDO = kTileBytes;
constexpr uint32_t kQOffK = 2 * kTileBytes;
constexpr uint32_t kQOffV = (2 + kKStages) * kTileBytes;
constexpr uint32_t kQSmem = (2 + kKStages + kVStages) * kTileBytes + 1024;

struct DqBarriers {
  uint64_t q_full, q_empty;
  uint64_t k_full[kKStages], k_empty[kKStages];
  uint64_t v_full[kVStages], v_empty[kVStages];
  uint64_t s_full, s_consumed;
  uint64_t dp_full[2], ds_ready[2], dq_done[2];
  uint64_t acc_done, drain[3];
};

// A dQ work item: one 128-row query tile (b, query head h, group g, tile qt).
struct DqItem {
  int b, h, kvh, g, qt, nkv, mq0;
  bool sh;
};

__device__ __forceinline__ DqItem decode_dq_item(const Params& p, int item) {
  const int T = p.G / kTile, ng = p.N / p.G, R = p.Hq / p.Hkv;
  // the query tiles of all query heads of a few (b, kv head, group) units run together
  // (they share K and V through L2), heaviest query tiles first
  int inner, bkg;
  chunked_lpt(item, p.B * p.Hkv * ng, T * R, bkg, inner);
  DqItem it;
  it.qt = T - 1 - inner / R;
  it.g = bkg % ng;
  const int bk = bkg / ng;
  it.kvh = bk % p.Hkv;
  it.b = bk / p.Hkv;
  it.h = it.kvh * R + inner % R;
  it.sh = q_head_shifted(it.h, p);
  it.nkv = p.causal ? it.qt + 1 : T;
  it.mq0 = src_row(it.g * p.G + it.qt * kTile, it.sh, p.G, p.N);
  return it;
}

// q_empty completes once both Q/dO readers (the S and dP issuers) are done with an item and
// every other role has read the item's slot; no role can then fall two items behind the
// producer, so every parity wait on q_full sees the phase it means.
constexpr uint32_t kDqQEmptyArrivals = 1 + 1 + 1 + kMathThreads / 32;

// Persistent: one CTA per SM takes query tiles from a counter in the workspace (zeroed by
// the row-sum pass in front of it). Three MMA issuers, one thread each (a thread issues a
// tcgen05.mma only every ~45 cycles, against 64 cycles of tensor work per 128 x 128 x 16
// MMA, and slower still while math warps share its scheduler; the dQ pass has 24 MMAs per
// key tile):
//   warp 1 (TMEM owner): S(j) = Q K_j^T into TMEM [0,128) once the math warps hold S(j-1)
//            in registers;
//   warp 2:  dP(j) = dO V_j^T into buffer j % 2 ([128,256) / [256,384)) once dQ(j-2) has
//            read the dS that buffer held;
//   warp 3:  dQ += dS(j) K_j ([384,512)) once the math warps published dS(j).
// With dP double-buffered, S and dP of key tile j+1 are computed while the math warps work
// on tile j, so the math never waits for the tensor cores in the steady state. The rings
// (K, V, S, dP) run on across the items of a CTA, so the next tile's S and dP are computed
// while the math warps write the current tile's dq.
__global__ void __launch_bounds__(kThreads, 1)
    tc_dq_kernel(const Params p, const __grid_constant__ CUtensorMap tm_q,
                 const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                 const __grid_constant__ CUtensorMap tm_do, int nitems) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  __shared__ DqBarriers bars;
  __shared__ uint32_t tmem_base_sh;
  __shared__ AbortState abort_state;
  __shared__ int item_slot[2];  // the CTA's k-th item in slot k & 1 (-1: no more work)

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  unsigned* const next_item = p.status + kDqWorkCounter;

  const Abort ab{smem_addr(&abort_state)};
  if (threadIdx.x == 0) {
    abort_state_init(abort_state, p.status, p.wait_limit_ns, 0);
    mbar_init(smem_addr(&bars.q_full), 1);
    mbar_init(smem_addr(&bars.q_empty), kDqQEmptyArrivals);
    for (int s = 0; s < kKStages; s++) {
      mbar_init(smem_addr(&bars.k_full[s]), 1);
      mbar_init(smem_addr(&bars.k_empty[s]), 2);  // S(j) and dQ(j) both read K_j
    }
    for (int s = 0; s < kVStages; s++) {
      mbar_init(smem_addr(&bars.v_full[s]), 1);
      mbar_init(smem_addr(&bars.v_empty[s]), 1);
    }
    mbar_init(smem_addr(&bars.s_full), 1);
    mbar_init(smem_addr(&bars.s_consumed), kMathThreads);
    for (int s = 0; s < 2; s++) {
      mbar_init(smem_addr(&bars.ds_ready[s]), kMathThreads);
      mbar_init(smem_addr(&bars.dp_full[s]), 1);
      mbar_init(smem_addr(&bars.dq_done[s]), 1);
    }
    for (int s = 0; s < 3; s++) mbar_init(smem_addr(&bars.drain[s]), 1);
    mbar_init(smem_addr(&bars.acc_done), 1);
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(smem_addr(&tmem_base_sh), kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  const uint32_t colS = 0, colDP = 128, colDQ = 384;  // dP buffers at colDP, colDP + 128
  const uint32_t sQ = smem_addr(smem + kQOffQ), sDO = smem_addr(smem + kQOffDO);
  const uint32_t qfull = smem_addr(&bars.q_full), qempty = smem_addr(&bars.q_empty);

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      int nk = 0, nv = 0;   // K and V tiles loaded so far (ring positions)
      int q_last = -1;      // item index (k) of the latest Q/dO load, -1 after the stop
      for (int k = 0, ok = 1; ok; k++) {
        int item = (int)atomicAdd(next_item, 1u);
        // stop when the work is done or a CTA of this launch gave up
        if (item >= nitems || *reinterpret_cast<volatile unsigned*>(p.status) != 0u) item = -1;
        if (k > 0 && !mbar_wait(qempty, (k - 1) & 1, ab)) break;
        item_slot[k & 1] = item;
        if (item < 0) {
          mbar_arrive(qfull);  // completes the phase: every role reads -1 and stops
          q_last = -1;
          break;
        }
        const DqItem it = decode_dq_item(p, item);
        mbar_arrive_expect_tx(qfull, 2 * kTileBytes);
        const int qrow = (it.b * p.Hq + it.h) * p.N + it.mq0;
        tma_load_2d(sQ, &tm_q, qfull, 0, qrow);
        tma_load_2d(sQ + kBoxBytes, &tm_q, qfull, 64, qrow);
        tma_load_3d(sDO, &tm_do, qfull, 0, it.h, it.b * p.N + it.mq0);
        tma_load_3d(sDO + kBoxBytes, &tm_do, qfull, 64, it.h, it.b * p.N + it.mq0);
        q_last = k;
        for (int j = 0; j < it.nkv; j++) {
          const int mk = src_row(it.g * p.G + j * kTile, it.sh, p.G, p.N);
          const int krow = (it.b * p.Hkv + it.kvh) * p.N + mk;
          const int sk = nk % kKStages, sv = nv % kVStages;
          if (!mbar_wait(smem_addr(&bars.k_empty[sk]), ((nk / kKStages) & 1) ^ 1, ab)) {
            ok = 0;
            break;
          }
          const uint32_t kb = smem_addr(&bars.k_full[sk]);
          const uint32_t sKs = smem_addr(smem + kQOffK + sk * kTileBytes);
          mbar_arrive_expect_tx(kb, kTileBytes);
          tma_load_2d(sKs, &tm_k, kb, 0, krow);
          tma_load_2d(sKs + kBoxBytes, &tm_k, kb, 64, krow);
          nk++;
          if (!mbar_wait(smem_addr(&bars.v_empty[sv]), ((nv / kVStages) & 1) ^ 1, ab)) {
            ok = 0;
            break;
          }
          const uint32_t vb = smem_addr(&bars.v_full[sv]);
          const uint32_t sVs = smem_addr(smem + kQOffV + sv * kTileBytes);
          mbar_arrive_expect_tx(vb, kTileBytes);
          tma_load_3d(sVs, &tm_v, vb, 0, it.kvh, it.b * p.N + mk);
          tma_load_3d(sVs + kBoxBytes, &tm_v, vb, 64, it.kvh, it.b * p.N + mk);
          nv++;
        }
      }
      // the last load into each ring stage (the latest phase of its barrier) and a Q/dO load
      // not yet consumed land before the CTA can exit (own time limit, no abort)
      for (int t = nk - 1; t >= 0 && t >= nk - kKStages; t--)
        mbar_wait_drain(smem_addr(&bars.k_full[t % kKStages]), (t / kKStages) & 1, p.status,
                        p.wait_limit_ns);
      for (int t = nv - 1; t >= 0 && t >= nv - kVStages; t--)
        mbar_wait_drain(smem_addr(&bars.v_full[t % kVStages]), (t / kVStages) & 1, p.status,
                        p.wait_limit_ns);
      if (q_last >= 0) mbar_wait_drain(qfull, q_last & 1, p.status, p.wait_limit_ns);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer: S
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16_f32(kTile, kTile, false, false);
      // Descriptors are built once; a stage or a k-step only adds a constant to the start
      // address field (bytes / 16; shared memory stays below 256 KB, so nothing carries out).
      const uint64_t dQd = smem_desc_sw128(sQ, 16, 1024);
      const uint64_t dK0 = smem_desc_sw128(smem_addr(smem + kQOffK), 16, 1024);
      int gs = 0;  // S tiles issued (all items)
      bool ok = true;
      for (int k = 0; ok; k++) {
        if (!mbar_wait(qfull, k & 1, ab)) break;
        const int item = item_slot[k & 1];
        if (item < 0) break;
        const int nkv = decode_dq_item(p, item).nkv;
        tc_fence_after();
        for (int j = 0; j < nkv; j++, gs++) {
          // S = Q K_j^T, once the math warps hold the previous S in registers
          if (gs >= 1 && !mbar_wait(smem_addr(&bars.s_consumed), (gs - 1) & 1, ab)) {
            ok = false;
            break;
          }
          const int sk = gs % kKStages;
          if (!mbar_wait(smem_addr(&bars.k_full[sk]), (gs / kKStages) & 1, ab)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t dk = opaque64(dK0) + (uint64_t)(sk * kTileDesc);
          const uint64_t dq = opaque64(dQd);
#pragma unroll
          for (int kk = 0; kk < kD / 16; kk++)
            mma_ss(tmem + colS, dq + kmajor_koff(kk), dk + kmajor_koff(kk), idesc_s, kk > 0);
          mma_commit(smem_addr(&bars.s_full));
          mma_commit(smem_addr(&bars.k_empty[sk]));
        }
        if (ok) mma_commit(qempty);  // Q is no longer read once these S have completed
      }
      mma_commit(smem_addr(&bars.drain[0]));
      mbar_wait_drain(smem_addr(&bars.drain[0]), 0, p.status, p.wait_limit_ns);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------------ MMA issuer: dP
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16_f32(kTile, kTile, false, false);
      const uint64_t dDOd = smem_desc_sw128(sDO, 16, 1024);
      const uint64_t dV0 = smem_desc_sw128(smem_addr(smem + kQOffV), 16, 1024);
      int gd = 0;  // dP tiles issued (all items); buffer gd % 2
      bool ok = true;
      for (int k = 0; ok; k++) {
        if (!mbar_wait(qfull, k & 1, ab)) break;
        const int item = item_slot[k & 1];
        if (item < 0) break;
        const int nkv = decode_dq_item(p, item).nkv;
        tc_fence_after();
        for (int j = 0; j < nkv; j++, gd++) {
          // dP = dO V_j^T into buffer gd % 2, once the dQ MMA two tiles back has read it
          if (gd >= 2 &&
              !mbar_wait(smem_addr(&bars.dq_done[gd & 1]), ((gd - 2) >> 1) & 1, ab)) {
            ok = false;
            break;
          }
          const int sv = gd % kVStages;
          if (!mbar_wait(smem_addr(&bars.v_full[sv]), (gd / kVStages) & 1, ab)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t dv = opaque64(dV0) + (uint64_t)(sv * kTileDesc);
          const uint64_t ddo = opaque64(dDOd);
#pragma unroll
          for (int kk = 0; kk < kD / 16; kk++)
            mma_ss(tmem + colDP + (gd & 1) * 128, ddo + kmajor_koff(kk), dv + kmajor_koff(kk),
                   idesc_s, kk > 0);
          mma_commit(smem_addr(&bars.dp_full[gd & 1]));
          mma_commit(smem_addr(&bars.v_empty[sv]));
        }
        if (ok) mma_commit(qempty);  // dO is no longer read once these dP have completed
      }
      mma_commit(smem_addr(&bars.drain[1]));
      mbar_wait_drain(smem_addr(&bars.drain[1]), 0, p.status, p.wait_limit_ns);
    }
  } else if (warp == 3) {
    // ------------------------------------------------------------------ MMA issuer: dQ
    if (lane == 0) {
      const uint32_t idesc_g = idesc_bf16_f32(kTile, kD, false, true);
      const uint64_t dKm0 = smem_desc_sw128(smem_addr(smem + kQOffK), kBoxBytes, 1024);
      int gq = 0;  // dQ steps issued (all items)
      bool ok = true;
      for (int k = 0; ok; k++) {
        if (!mbar_wait(qfull, k & 1, ab)) break;
        const int item = item_slot[k & 1];
        if (item < 0) break;
        mbar_arrive(qempty);  // slot read
        const int nkv = decode_dq_item(p, item).nkv;
        for (int j = 0; j < nkv; j++, gq++) {
          // dQ += dS K_j, dS read from dP buffer gq % 2
          if (!mbar_wait(smem_addr(&bars.ds_ready[gq & 1]), (gq >> 1) & 1, ab)) {
            ok = false;
            break;
          }
          const int sk = gq % kKStages;
          if (!mbar_wait(smem_addr(&bars.k_full[sk]), (gq / kKStages) & 1, ab)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t dkm = opaque64(dKm0) + (uint64_t)(sk * kTileDesc);
          const uint32_t acc0 = j > 0;
#pragma unroll
          for (int kk = 0; kk < kTile / 16; kk++)
            mma_ts(tmem + colDQ, tmem + packed_col(colDP + (gq & 1) * 128, kk),
                   dkm + mn_koff(kk), idesc_g, kk ? 1u : acc0);
          mma_commit(smem_addr(&bars.dq_done[gq & 1]));
          mma_commit(smem_addr(&bars.k_empty[sk]));
        }
        if (ok) mma_commit(smem_addr(&bars.acc_done));
      }
      mma_commit(smem_addr(&bars.drain[2]));
      mbar_wait_drain(smem_addr(&bars.drain[2]), 0, p.status, p.wait_limit_ns);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------------ per query row math
    const int quarter = warp & 3;
    const int c0 = ((warp - 4) >> 2) * 64;  // this warp's 64 key columns of the tile
    const int row = quarter * 32 + lane;    // query row inside the tile
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_off + colS + c0;
    const float sl2 = p.scale_log2;
    const uint64_t sl2x2 = f2pack(sl2, sl2);
    uint32_t gm = 0;  // key tiles processed (all items)
    for (int k = 0;; k++) {
      bool ok = mbar_wait(qfull, k & 1, ab);
      __syncwarp();
      if (!__all_sync(0xffffffffu, ok)) break;
      const int item = item_slot[k & 1];
      if (item < 0) break;
      if (lane == 0) mbar_arrive(qempty);  // slot read
      const DqItem it = decode_dq_item(p, item);
      const int m = src_row(it.g * p.G + it.qt * kTile + row, it.sh, p.G, p.N);
      const size_t lrow = ((size_t)it.b * p.Hq + it.h) * p.N + m;
      const float nlse2 = -p.lse[lrow] * kLog2e;
      const float Dm = p.Dsum[lrow];
      const uint64_t nlse2x2 = f2pack(nlse2, nlse2), Dmx2 = f2pack(Dm, Dm);
      for (int j = 0; j < it.nkv; j++, gm++) {
        ok = mbar_wait(smem_addr(&bars.s_full), gm & 1, ab);
        __syncwarp();
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        tc_fence_after();
        const bool diag = p.causal && j == it.qt;
        float pr[64];
        {
          uint32_t x0[32], x1[32];
          tmem_ld32(tS, x0);
          tmem_ld32(tS + 32, x1);
          tmem_wait_ld();
          tc_fence_before();
          mbar_arrive(smem_addr(&bars.s_consumed));  // S may now be overwritten
          if (diag) {
            mask_scores(x0, x1, row - c0, 1);  // key column after the query row: P = 0
#pragma unroll
            for (int c = 0; c < 64; c += 2) {
              float a0, a1;
              f2unpack(ffma2(score_pair(x0, x1, c), sl2x2, nlse2x2), a0, a1);
              pr[c] = fast_exp2(a0);
              pr[c + 1] = fast_exp2(a1);
            }
          } else {
#pragma unroll
            for (int c = 0; c < 64; c += 2) {
              const uint64_t a = ffma2(score_pair(x0, x1, c), sl2x2, nlse2x2);
              if ((kDqPolyMask >> (c >> 1)) & 1u) {
                f2unpack(exp2_poly2(a), pr[c], pr[c + 1]);
              } else {
                float a0, a1;
                f2unpack(a, a0, a1);
                pr[c] = fast_exp2(a0);
                pr[c + 1] = fast_exp2(a1);
              }
            }
          }
          pin_regs(pr);
        }
        ok = mbar_wait(smem_addr(&bars.dp_full[gm & 1]), (gm >> 1) & 1, ab);
        __syncwarp();
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        tc_fence_after();
        {
          const uint32_t tDP = tmem + lane_off + colDP + (gm & 1) * 128 + c0;
          uint32_t x0[32], x1[32];
          tmem_ld32(tDP, x0);
          tmem_ld32(tDP + 32, x1);
          tmem_wait_ld();
#pragma unroll
          for (int ch = 0; ch < 2; ch++) {
            uint32_t pk[16];
#pragma unroll
            for (int t = 0; t < 16; t++) {
              const int c = ch * 32 + 2 * t;
              float s0, s1;
              f2unpack(fmul2(f2pack(pr[c], pr[c + 1]), fsub2(score_pair(x0, x1, c), Dmx2)), s0,
                       s1);
              pk[t] = pack_bf16x2(s0, s1);
            }
            tmem_st16(tDP + ch * 16, pk);  // dS of these 64 key columns, over dP already read
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(smem_addr(&bars.ds_ready[gm & 1]));
      }
      if (!ok) break;
      ok = mbar_wait(smem_addr(&bars.acc_done), k & 1, ab);
      __syncwarp();
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      // The fp32 accumulator is transposed first (8 x 8 chunks of four values within each
      // group of eight lanes, per 32 columns): lane 8g + i then holds columns 4i .. 4i + 3
      // of each 32-column block for the group's eight rows, so that its (cos, sin) entries
      // (two pairs per row and block) are read 128 contiguous bytes per eight lanes and its
      // stores are 64 contiguous bytes per eight lanes. The tile's rows are consecutive
      // tokens from m - row (a 128-row tile never straddles the roll's wrap).
      const int l8 = lane & 7;
      const size_t tok0 = (size_t)(m - row + (row & ~7));  // token of the group's first row
      uint32_t w[32];  // bf16 pairs: block ch, row c of the group -> w[16ch + 2c], w[16ch + 2c + 1]
#pragma unroll
      for (int ch = 0; ch < 2; ch++) {
        uint32_t x[32];
        tmem_ld32(tmem + lane_off + colDQ + c0 + ch * 32, x);
        tmem_wait_ld();
        transpose_chunks8(x, lane);
        const float4* cs4 =
            reinterpret_cast<const float4*>(p.cs + tok0 * (kD / 2) + (c0 + 32 * ch) / 2 + 2 * l8);
#pragma unroll
        for (int c = 0; c < 8; c++) {
          const float4 cs = cs4[c * (kD / 4)];  // pairs 2 l8, 2 l8 + 1 of row c of the group
#pragma unroll
          for (int e = 0; e < 2; e++) {
            const float cc = e ? cs.z : cs.x, sn = e ? cs.w : cs.y;
            const float x0 = __uint_as_float(x[4 * c + 2 * e]) * p.scale;
            const float x1 = __uint_as_float(x[4 * c + 2 * e + 1]) * p.scale;
            w[16 * ch + 2 * c + e] = pack_bf16x2(fmaf(x0, cc, x1 * sn), fmaf(-x0, sn, x1 * cc));
          }
        }
      }
      __nv_bfloat16* dq = static_cast<__nv_bfloat16*>(p.dq) +
                          ((size_t)it.b * p.N + tok0) * p.Hq * kD + (size_t)it.h * kD + c0 + 4 * l8;
#pragma unroll
      for (int c = 0; c < 8; c++)
#pragma unroll
        for (int ch = 0; ch < 2; ch++)
          *reinterpret_cast<uint2*>(dq + (size_t)c * p.Hq * kD + 32 * ch) =
              make_uint2(w[16 * ch + 2 * c], w[16 * ch + 2 * c + 1]);
      // the next item's first dQ MMA overwrites the accumulator only after this item's
      // dS of its first key tile, which these warps publish after the loads above
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
  CUtensorMap tq, tk, tv, tdo, tterms, tcs, tdk, tdv;
  cudaError_t e = make_bwd_maps(p, &tq, &tk, &tv, &tdo);
  if (e) return e;
  // row terms: rows of 16 bf16 (32 bytes), one per (b, query head, token), 32-byte swizzle
  if ((e = make_tmap_2d(&tterms, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, CU_TENSOR_MAP_SWIZZLE_32B,
                        p.rowterms, 16, (uint64_t)p.B * p.Hq * p.N, 32, 16, kTile)))
    return e;
  // (cos, sin) table: one row of d floats per token, boxes of 32 floats x 128 tokens
  if ((e = make_tmap_2d(&tcs, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, CU_TENSOR_MAP_SWIZZLE_128B, p.cs,
                        kD, (uint64_t)p.N, kD * 4, 32, kTile)))
    return e;
  if ((e = make_tmap_bf16_3d(&tdk, p.dk, kD, p.Hkv, (uint64_t)p.B * p.N, kD * 2,
                             (uint64_t)p.Hkv * kD * 2, 64, kTile)))
    return e;
  if ((e = make_tmap_bf16_3d(&tdv, p.dv, kD, p.Hkv, (uint64_t)p.B * p.N, kD * 2,
                             (uint64_t)p.Hkv * kD * 2, 64, kTile)))
    return e;
  if ((e = cudaFuncSetAttribute(tc_dkdv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)kKVSmem)))
    return e;
  const long tiles = (long)p.B * p.Hkv * (p.N / p.G) * (p.G / kTile);
  tc_dkdv_kernel<<<dim3((unsigned)tiles), dim3(kThreads), kKVSmem, st>>>(p, tq, tk, tv, tdo,
                                                                        tterms, tcs, tdk, tdv);
  return cudaGetLastError();
}

cudaError_t launch_tc_bwd_dq(const Params& p, cudaStream_t st) {
  CUtensorMap tq, tk, tv, tdo;
  cudaError_t e = make_bwd_maps(p, &tq, &tk, &tv, &tdo);
  if (e) return e;
  if ((e = cudaFuncSetAttribute(tc_dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)kQSmem)))
    return e;
  // persistent: at most one CTA per SM (one fits), each taking query tiles until none is left
  const long tiles = (long)p.B * p.Hq * (p.N / p.G) * (p.G / kTile);
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev))) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev))) return e;
  const unsigned grid = (unsigned)(tiles < sms ? tiles : sms);
  tc_dq_kernel<<<dim3(grid), dim3(kThreads), kQSmem, st>>>(p, tq, tk, tv, tdo, (int)tiles);
  return cudaGetLastError();
}

}  // namespace s2
