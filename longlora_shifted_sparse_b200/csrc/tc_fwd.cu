// S2-Attn forward on the 5th-generation tensor cores (tcgen05, TMEM accumulators, TMA).
//
// Work item = two consecutive 128-row query tiles (A = 2p, B = 2p+1) of one (batch, query
// head, group): rolled rows g*G + 256p ... + 255. A shifted head's rolled row r is token
// (r + G/2) mod N, and because G/2 is a multiple of 128 a tile never straddles the wrap,
// so the -G/2 roll of q, k, v and the +G/2 roll back of o are just the row coordinate of
// each TMA load / store ("LongLoRA and Shifted Sparse Attention (S^2-Attn)", definition;
// "LongLoRA: Efficient 100k Context LLM Fine-Tuning Guide", Implementation, Step 1).
// Inside the group each query tile attends to key tiles 0..its own index (causal: tiles
// above the diagonal are skipped, the diagonal tile is masked on group-local positions).
//
// Roles (640 threads, five warpgroups):
//   warp 0       TMA producer: per work item Q_A, K_0, Q_B, then V_0, K_j, V_j into two
//                2-stage rings (each K/V tile serves both query tiles; the rings run on
//                across the items of a CTA). Q_A and Q_B have a buffer each.
//   warp 1       MMA issuer (the warp runs the loop, one elected lane issues) and TMEM
//                owner. Order per key tile j: PV_A(j-1), QK_A(j), PV_B(j-1), QK_B(j): while
//                the tensor cores work on one tile, the other tile's softmax runs
//                (ping-pong). The ping-pong runs on across a CTA's items: an item's last
//                PVs go out in the next item's first step, after its QK_A(0).
//   warps 2, 3   idle (they complete warpgroup 0, whose registers go to the softmax).
//   warps 4..11  softmax of tile A; warps 12..19 softmax of tile B. A query row (= TMEM
//                lane) is shared by two warps, one per 64-column half of S: each loads its
//                half once, takes the partial max, swaps it with its partner through shared
//                memory (a 64-thread named barrier), and writes P = exp2(S log2(e)/sqrt(d)
//                - m) as bf16 over the first 32 columns of its half (scale-and-shift and
//                row sums on packed fp32 pairs, the row max with three-input max). Four softmax warps per
//                scheduler hide the TMEM-load and MUFU latencies that bound a one-warp-per-
//                row softmax. The O accumulator (TMEM) is rescaled only when the running max
//                grows by more than 2^8; the stale max keeps every P <= 256 and l uses the
//                same max. When S_t(j) has landed, PV_t(j-1) has completed (commit order),
//                so the rescale needs no extra wait. Epilogue: each half stores its 64
//                columns of O / l (l = sum of both partial sums) as bf16 at the token's
//                original row, whole 128-byte row segments per store after a shuffle
//                transpose within groups of eight lanes; LSE = ln 2 * (m + log2 l).
// TMEM: S_A [0,128), S_B [128,256), O_A [256,384), O_B [384,512).
// Persistent CTAs (one per SM) take work items from a counter in the workspace. Items are
// numbered a chunk of (b, kv head, group) units at a time, the heaviest tile pairs of those
// units first, so the items in flight reuse K and V from L2 and the last items are light.
// Between two items of a CTA the producer and the issuer run ahead: the next item's Q_A
// loads once the last QK^T of the current tile A has completed (and every softmax warp has
// taken the current item's id), its Q_B once tile B's has, and its first QK^T MMAs run
// while the softmax warps finish the current item.
// Every wait is bounded; on expiry the CTA records it in the status word and drains.
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
constexpr uint32_t kTileBytes = kTile * kD * 2;    // 32 KB: 128 rows x 128 bf16
constexpr uint32_t kHalfBytes = kTileBytes / 2;    // one 128 x 64 TMA box
// 20 warps: TMA, MMA, two idle, 16 softmax warps. Five warps share one scheduler's 64K-byte
// register file, so a launch hands each thread 96 registers. Warpgroup 0 then drops to
// kRegsOther and the four softmax warpgroups rise to kRegsSoftmax (setmaxnreg), enough to
// hold their 64 scores per row without spilling. The split must fit the launch allocation
// (an increase beyond it would wait forever), which the launcher checks before every launch.
constexpr int kThreads = 640;
constexpr int kRegsOther = 64, kRegsSoftmax = 104;
static_assert(128 * kRegsOther + (kThreads - 128) * kRegsSoftmax <= kThreads * 96,
              "register split exceeds the launch allocation");
constexpr int kSoftmaxThreadsPerTile = 256;
constexpr int kSoftmaxWarps = 2 * kSoftmaxThreadsPerTile / 32;
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;          // log2 units

// Column pairs (bit c2 of a 16-bit mask, per 32-column chunk) whose exponentials go to the
// FMA-pipe exp2 (packed pairs) instead of the MUFU unit. At d = 128 the MUFU needs as many
// cycles per key tile as the tensor cores. On a B200 moving 25% / 37.5% / 50% of the
// exponentials to the scalar form of the polynomial slowed the 32k forward from 2.32 ms to
// 2.52 / 2.84 / 3.10 ms; with the packed form, 12.5% / 25% / 31% gave 2.08 / 2.09 / 2.14 ms
// against 2.04-2.05 ms with none. So every exponential stays on the MUFU unless a build
// overrides this mask.
#ifndef S2_FWD_POLY_MASK
#define S2_FWD_POLY_MASK 0x0000u
#endif
constexpr unsigned kPolyMask = S2_FWD_POLY_MASK;

// dynamic shared memory: Q_A Q_B | K0 K1 | V0 V1, each 32 KB, 1024-byte aligned
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = 2 * kTileBytes;
constexpr uint32_t kOffV = 4 * kTileBytes;
constexpr uint32_t kSmemBytes = 6 * kTileBytes + 1024;

struct FwdBarriers {
  uint64_t q_full[2], q_empty[2];                 // per query tile; q_full[0] also publishes the item
  uint64_t k_full[2], k_empty[2];
  uint64_t v_full[2], v_empty[2];
  uint64_t s_full[2], p_full[2], o_final[2];  // index: query tile A = 0, B = 1
  uint64_t drain;
};

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint64_t opaque64(uint64_t v) {
  uint64_t r;
  asm volatile("mov.b64 %0, %1;" : "=l"(r) : "l"(v));
  return r;
}

// Max of a thread's 64 scores, as a tree of three-input maxima (short dependency chain).
__device__ __forceinline__ float max64(const uint32_t (&x0)[32], const uint32_t (&x1)[32]) {
  float v[64];
#pragma unroll
  for (int c = 0; c < 32; c++) {
    v[c] = __uint_as_float(x0[c]);
    v[32 + c] = __uint_as_float(x1[c]);
  }
  float m1[22];
#pragma unroll
  for (int c = 0; c < 21; c++) m1[c] = fmax3(v[3 * c], v[3 * c + 1], v[3 * c + 2]);
  m1[21] = v[63];
  float m2[8];
#pragma unroll
  for (int c = 0; c < 7; c++) m2[c] = fmax3(m1[3 * c], m1[3 * c + 1], m1[3 * c + 2]);
  m2[7] = m1[21];
  return fmax3(fmax3(m2[0], m2[1], m2[2]), fmax3(m2[3], m2[4], m2[5]), fmaxf(m2[6], m2[7]));
}

// P = exp2(S * sl2 - m) for a thread's 64 scores, written as bf16 pairs over the first 32
// of its 64 TMEM columns of S (the PV MMA reads them from there); returns the sum of P.
// The scale-and-shift and the running sums (even and odd columns) use packed fp32 pairs.
__device__ __forceinline__ float write_p64(const uint32_t (&x0)[32], const uint32_t (&x1)[32],
                                           float sl2, float nm, uint32_t tS) {
  const uint64_t sl2x2 = f2pack(sl2, sl2), nmx2 = f2pack(nm, nm);
  uint64_t acc = f2pack(0.f, 0.f);
#pragma unroll
  for (int ch = 0; ch < 2; ch++) {
    uint32_t pk[16];
#pragma unroll
    for (int c2 = 0; c2 < 16; c2++) {
      const float s0 = __uint_as_float(ch ? x1[2 * c2] : x0[2 * c2]);
      const float s1 = __uint_as_float(ch ? x1[2 * c2 + 1] : x0[2 * c2 + 1]);
      const uint64_t a = ffma2(f2pack(s0, s1), sl2x2, nmx2);
      float p0, p1;
      if ((kPolyMask >> c2) & 1u) {
        f2unpack(exp2_poly2(a), p0, p1);
      } else {
        float a0, a1;
        f2unpack(a, a0, a1);
        p0 = fast_exp2(a0);
        p1 = fast_exp2(a1);
      }
      acc = fadd2(acc, f2pack(p0, p1));
      pk[c2] = pack_bf16x2(p0, p1);
    }
    tmem_st16(tS + ch * 16, pk);
  }
  float r0, r1;
  f2unpack(acc, r0, r1);
  return r0 + r1;
}

// Multiplies the 64 bf16 P values a thread wrote (32 packed columns) by a power of two,
// which is exact in bf16.
__device__ __forceinline__ void scale_p64(uint32_t tS, float f) {
  uint32_t x[32];
  tmem_ld32(tS, x);
  tmem_wait_ld();
#pragma unroll
  for (int c = 0; c < 32; c++)
    x[c] = pack_bf16x2(__uint_as_float(x[c] << 16) * f, __uint_as_float(x[c] & 0xffff0000u) * f);
  tmem_st32(tS, x);
}

// 2^k for an integral k <= 0 (k = -inf gives 0), exact.
__device__ __forceinline__ float exp2_int(float k) {
  return k < -126.f ? 0.f : __int_as_float((static_cast<int>(k) + 127) << 23);
}

// Loads the thread's 64 scores; on the diagonal tile the keys after the query (group-local
// positions) get -inf, so that their P is 0.
__device__ __forceinline__ void load_s64(uint32_t tS, bool diag, int first_col, int row,
                                         uint32_t (&x0)[32], uint32_t (&x1)[32]) {
  tmem_ld32(tS, x0);
  tmem_ld32(tS + 32, x1);
  tmem_wait_ld();
  if (diag) {
    const uint32_t ninf = 0xff800000u;
#pragma unroll
    for (int c = 0; c < 32; c++) {
      x0[c] = first_col + c <= row ? x0[c] : ninf;
      x1[c] = first_col + 32 + c <= row ? x1[c] : ninf;
    }
  }
}

// Units per chunk of the work order: as many (b, kv head, group) units as keep about
// kLptKVBudget bytes of K and V in flight, and at least kLptChunk. Short groups thus get
// wide chunks: with few key tiles per item, a chunk of only kLptChunk units would start its
// heaviest items late in the run and leave a long tail, while their K and V still fit L2.
#ifndef S2_FWD_LPT_BUDGET_MB
#define S2_FWD_LPT_BUDGET_MB 16
#endif
constexpr long long kLptKVBudget = (long long)S2_FWD_LPT_BUDGET_MB << 20;
__device__ __forceinline__ int fwd_lpt_chunk(const Params& p) {
  // kLptKVBudget / (K and V bytes of one group = 2 * G * d * 2), in 32-bit arithmetic
  const int c = (int)(kLptKVBudget / (4 * kD)) / p.G;
  return c > kLptChunk ? c : kLptChunk;
}

// A work item: two consecutive 128-row query tiles (A = qt0, B = qt0 + 1) of one
// (batch, query head, group). Items are numbered in the chunked longest-first order.
struct FwdItem {
  int b, h, kvh, g, qt0, nA, nB, r0;
  bool sh;
};

__device__ __forceinline__ FwdItem decode_item(const Params& p, int item) {
  const int T = p.G / kTile, ng = p.N / p.G, R = p.Hq / p.Hkv;
  int inner, bkg;
  chunked_lpt(item, p.B * p.Hkv * ng, (T / 2) * R, bkg, inner, fwd_lpt_chunk(p));
  FwdItem it;
  const int pr = T / 2 - 1 - inner / R;
  it.g = bkg % ng;
  const int bk = bkg / ng;
  it.kvh = bk % p.Hkv;
  it.b = bk / p.Hkv;
  it.h = it.kvh * R + inner % R;
  it.sh = q_head_shifted(it.h, p);
  it.qt0 = 2 * pr;
  it.nA = p.causal ? it.qt0 + 1 : T;   // key tiles of tile A
  it.nB = p.causal ? it.qt0 + 2 : T;   // key tiles of tile B (>= nA)
  it.r0 = it.g * p.G + it.qt0 * kTile; // rolled row of tile A's row 0
  return it;
}

// Persistent: one CTA per SM takes work items from a counter in the workspace (zeroed by
// the RoPE pass that precedes every forward) until none is left. While the softmax warps
// finish one item (last key tiles, epilogue), the producer already loads the next item's
// query tiles and key tiles and the issuer runs its first QK^T MMAs.
__global__ void __launch_bounds__(kThreads, 1)
    tc_fwd_kernel(const Params p, const __grid_constant__ CUtensorMap tm_q,
                  const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                  int nitems) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  __shared__ FwdBarriers bars;
  __shared__ uint32_t tmem_base_sh;
  __shared__ AbortState abort_state;
  // the CTA's k-th work item sits in slot k & 1 (-1: no more work), published with q_full[0]
  __shared__ int item_slot[2];
  // row-max exchange between the two warps that share a row: [parity][tile][half][row]
  __shared__ float xmax[2][2][2][kTile];
  __shared__ float xsum[2][kTile];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  unsigned* const next_item = p.status + kFwdWorkCounter;

  const Abort ab{smem_addr(&abort_state)};
  if (threadIdx.x == 0) {
    abort_state_init(abort_state, p.status, p.wait_limit_ns, 0);
    // Q_A is free once its last QK^T has completed (one commit) and every softmax warp has
    // read the item id (one arrival per warp): the next item's id is only published then, so
    // no softmax warp can fall two items behind the slot ring or the q_full[0] phases
    mbar_init(smem_addr(&bars.q_empty[0]), 1 + kSoftmaxWarps);
    mbar_init(smem_addr(&bars.q_empty[1]), 1);
    for (int s = 0; s < 2; s++) {
      mbar_init(smem_addr(&bars.q_full[s]), 1);
      mbar_init(smem_addr(&bars.k_full[s]), 1);
      mbar_init(smem_addr(&bars.k_empty[s]), 1);
      mbar_init(smem_addr(&bars.v_full[s]), 1);
      mbar_init(smem_addr(&bars.v_empty[s]), 1);
      mbar_init(smem_addr(&bars.s_full[s]), 1);
      mbar_init(smem_addr(&bars.p_full[s]), kSoftmaxThreadsPerTile);
      mbar_init(smem_addr(&bars.o_final[s]), 1);
    }
    mbar_init(smem_addr(&bars.drain), 1);
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(smem_addr(&tmem_base_sh), kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  const uint32_t sQ = smem_addr(smem + kOffQ);

  if (warp < 4) {
    // warpgroup 0 (TMA producer, MMA issuer, two idle warps) gives registers away
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsOther));
    if (warp == 0 && lane == 0) {
      // ------------------------------------------------------------------ TMA producer
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      int nk = 0, nv = 0;            // K and V tiles loaded so far (ring positions)
      int qa_last = -1, qb_last = -1;  // item index (k) of the latest Q_A / Q_B load
      for (int k = 0, ok = 1; ok; k++) {
        int item = (int)atomicAdd(next_item, 1u);
        // stop when the work is done or a CTA of this launch gave up
        if (item >= nitems || *reinterpret_cast<volatile unsigned*>(p.status) != 0u) item = -1;
        // Q_A of the previous item is no longer read and its id has been taken by all
        if (k > 0 && !mbar_wait(smem_addr(&bars.q_empty[0]), (k - 1) & 1, ab)) break;
        item_slot[k & 1] = item;
        const uint32_t qa = smem_addr(&bars.q_full[0]), qb = smem_addr(&bars.q_full[1]);
        if (item < 0) {
          mbar_arrive(qa);  // completes the phase: the consumers read -1 and stop
          qa_last = -1;     // (the previous Q_A has been read, so it has landed)
          break;
        }
        const FwdItem it = decode_item(p, item);
        const int qrow0 = (it.b * p.Hq + it.h) * p.N;
        mbar_arrive_expect_tx(qa, kTileBytes);
        tma_load_2d(sQ, &tm_q, qa, 0, qrow0 + src_row(it.r0, it.sh, p.G, p.N));
        tma_load_2d(sQ + kHalfBytes, &tm_q, qa, 64, qrow0 + src_row(it.r0, it.sh, p.G, p.N));
        qa_last = k;
        const int krow0 = (it.b * p.Hkv + it.kvh) * p.N;
        for (int j = 0; j < it.nB; j++) {
          const int s = nk & 1;
          const uint32_t ph = (nk >> 1) & 1;
          const int mk = src_row(it.g * p.G + j * kTile, it.sh, p.G, p.N);
          if (!mbar_wait(smem_addr(&bars.k_empty[s]), ph ^ 1, ab)) { ok = 0; break; }
          const uint32_t sK = smem_addr(smem + kOffK + s * kTileBytes);
          mbar_arrive_expect_tx(smem_addr(&bars.k_full[s]), kTileBytes);
          tma_load_2d(sK, &tm_k, smem_addr(&bars.k_full[s]), 0, krow0 + mk);
          tma_load_2d(sK + kHalfBytes, &tm_k, smem_addr(&bars.k_full[s]), 64, krow0 + mk);
          nk++;
          if (j == 0) {
            // Q_B after K_0: the next item's first QK^T (tile A) can start before this
            // item's tile B has finished with the previous Q_B
            if (k > 0 && !mbar_wait(smem_addr(&bars.q_empty[1]), (k - 1) & 1, ab)) {
              ok = 0;
              break;
            }
            const int qrow = qrow0 + src_row(it.r0 + kTile, it.sh, p.G, p.N);
            mbar_arrive_expect_tx(qb, kTileBytes);
            tma_load_2d(sQ + kTileBytes, &tm_q, qb, 0, qrow);
            tma_load_2d(sQ + kTileBytes + kHalfBytes, &tm_q, qb, 64, qrow);
            qb_last = k;
          }
          if (!mbar_wait(smem_addr(&bars.v_empty[s]), ph ^ 1, ab)) { ok = 0; break; }
          const uint32_t sV = smem_addr(smem + kOffV + s * kTileBytes);
          mbar_arrive_expect_tx(smem_addr(&bars.v_full[s]), kTileBytes);
          tma_load_3d(sV, &tm_v, smem_addr(&bars.v_full[s]), 0, it.kvh, it.b * p.N + mk);
          tma_load_3d(sV + kHalfBytes, &tm_v, smem_addr(&bars.v_full[s]), 64, it.kvh,
                      it.b * p.N + mk);
          nv++;
        }
      }
      // Let the loads in flight land before the CTA can exit: the last load into each ring
      // stage (the latest phase of its barrier) and query loads not yet consumed. These
      // waits ignore the abort flag (it may be set on this path) but keep their time limit.
      for (int t = nk - 1; t >= 0 && t >= nk - 2; t--)
        mbar_wait_drain(smem_addr(&bars.k_full[t & 1]), (t >> 1) & 1, p.status,
                        p.wait_limit_ns);
      for (int t = nv - 1; t >= 0 && t >= nv - 2; t--)
        mbar_wait_drain(smem_addr(&bars.v_full[t & 1]), (t >> 1) & 1, p.status,
                        p.wait_limit_ns);
      if (qa_last >= 0)
        mbar_wait_drain(smem_addr(&bars.q_full[0]), qa_last & 1, p.status, p.wait_limit_ns);
      if (qb_last >= 0)
        mbar_wait_drain(smem_addr(&bars.q_full[1]), qb_last & 1, p.status, p.wait_limit_ns);
    } else if (warp == 1) {
      // ------------------------------------------------------------------ MMA issuer
      // The whole warp runs the issue loop (warp-uniform control flow and descriptors);
      // one elected lane issues each MMA and commit.
      const uint32_t idesc_qk = idesc_bf16_f32(kTile, kTile, false, false);
      const uint32_t idesc_pv = idesc_bf16_f32(kTile, kD, false, true);
      // Descriptors are built once; a k-step or a stage only adds a constant to the start
      // address field (bytes / 16; every address stays below 256 KB, so no carry leaves it).
      // One thread issues every MMA while four softmax warps share its scheduler, so the
      // issue path is kept to a few instructions per MMA.
      const uint64_t dQ = smem_desc_sw128(sQ, 16, 1024);
      const uint64_t dK = smem_desc_sw128(smem_addr(smem + kOffK), 16, 1024);
      const uint64_t dV = smem_desc_sw128(smem_addr(smem + kOffV), kHalfBytes, 1024);
      constexpr uint32_t kTileDesc = kTileBytes >> 4;
      // Items run back to back in one ping-pong: an item's last PVs (key tile nB - 1) go out
      // in the next item's first step, after its QK_A(0) and before its QK_B(0), so the
      // tensor cores work on the next item while tile B's last softmax runs. Key tile j - 1
      // of step j = 0 is then the previous item's last (ring position kv - 1); a flush step
      // after the last item issues its final PVs.
      int kv = 0;                        // ring position of the item's key tile 0
      bool ok = true;
      int k = 0;
      for (;; k++) {
        if (!__all_sync(0xffffffffu, mbar_wait(smem_addr(&bars.q_full[0]), k & 1, ab))) {
          ok = false;
          break;
        }
        const int item = item_slot[k & 1];
        const bool flush = item < 0;     // no more items: only the previous item's PVs
        if (flush && k == 0) break;
        const FwdItem it = decode_item(p, flush ? 0 : item);
        const int nA = flush ? 0 : it.nA, nB = flush ? 1 : it.nB;
        tc_fence_after();
        for (int j = 0; j < nB; j++) {
          const int gj = kv + j, gjj = gj - 1;   // ring positions of key tiles j and j - 1
          const bool pv = j > 0 || k > 0;        // step j has PVs (of key tile j - 1)
          // V_{j-1} before the first PV, K_j only before the first QK^T: a PV never waits
          // for the key tile that follows it
          if (pv && !__all_sync(0xffffffffu, mbar_wait(smem_addr(&bars.v_full[gjj & 1]),
                                                       (gjj >> 1) & 1, ab))) {
            ok = false;
            break;
          }
          bool k_ready = false;
          tc_fence_after();
          // opaque per-iteration bases: the per-k-step descriptors are formed by one add at
          // their MMA instead of being hoisted out of the loop into (spilled) registers
          const uint64_t dKj = opaque64(dK) + (uint64_t)((gj & 1) * kTileDesc);
          const uint64_t dVj = opaque64(dV) + (uint64_t)((gjj & 1) * kTileDesc);
          const uint64_t dQj = opaque64(dQ);
#pragma unroll
          for (int t = 0; t < 2; t++) {
            const int nt = t ? nB : nA;
            const uint32_t tS = tmem + t * 128, tO = tmem + 256 + t * 128;
            // PV of key tile j - 1: inside the item while j - 1 < nt; at j = 0 the previous
            // item's last one (tile B always, tile A when not causal: it has nB key tiles)
            if (j > 0 ? j - 1 < nt : (k > 0 && (t == 1 || !p.causal))) {
              // p_full phases tile t consumed before: its key tiles in the earlier items
              // plus j - 1 (tile B has nB per item, kv in all; causal tile A one less each)
              const int pdone = t || !p.causal ? gjj : gjj - k;
              if (!__all_sync(0xffffffffu,
                              mbar_wait(smem_addr(&bars.p_full[t]), pdone & 1, ab))) {
                ok = false;
                break;
              }
              tc_fence_after();
              const uint32_t acc0 = j != 1;  // only an item's key tile 0 starts O afresh
#pragma unroll
              for (int kk = 0; kk < kTile / 16; kk++)  // P of key rows 64h.. at column 64h;
                mma_ts_elect(tO, tS + (kk >> 2) * 64 + (kk & 3) * 8,  // V k-step = 16 rows
                       dVj + (uint64_t)(kk * (2048 >> 4)), idesc_pv, kk ? 1u : acc0);
              if (j == 0 || j == nt) mma_commit_elect(smem_addr(&bars.o_final[t]));
            }
            // V_{j-1} is free once the last PV that reads it has been issued (tile B's)
            if (t == 1 && pv) mma_commit_elect(smem_addr(&bars.v_empty[gjj & 1]));
            if (j < nt && !flush) {
              // K_j before the step's first QK^T; Q_B before the item's first QK^T of tile B
              // (K_0 is ready by then: every item has a QK_A(0), so one wait covers both)
              const bool need_qb = t == 1 && j == 0;
              if (!k_ready || need_qb) {
                const uint32_t bar = need_qb ? smem_addr(&bars.q_full[1])
                                             : smem_addr(&bars.k_full[gj & 1]);
                const uint32_t par = need_qb ? (uint32_t)(k & 1) : (uint32_t)((gj >> 1) & 1);
                if (!__all_sync(0xffffffffu, mbar_wait(bar, par, ab))) {
                  ok = false;
                  break;
                }
                k_ready = true;
              }
              tc_fence_after();
              const uint64_t dQt = dQj + (uint64_t)(t * kTileDesc);
#pragma unroll
              for (int kk = 0; kk < kD / 16; kk++) {
                const uint64_t koff =
                    (uint64_t)(((kk >> 2) * kHalfBytes + (kk & 3) * 32) >> 4);
                mma_ss_elect(tS, dQt + koff, dKj + koff, idesc_qk, kk > 0);
              }
              // failure-path self-test: CTA 0 withholds the arrival of score tile B at key
              // tile 1 of its first item (every item's tile B has at least two key tiles),
              // so that tile's softmax warps and then this thread wait in vain until the limit
              if (!(p.inject == kInjectFwd && blockIdx.x == 0 && k == 0 && t == 1 && j == 1))
                mma_commit_elect(smem_addr(&bars.s_full[t]));
              // Q_t is free after the last QK^T that reads it
              if (j == nt - 1) mma_commit_elect(smem_addr(&bars.q_empty[t]));
            }
          }
          if (!ok) break;
          if (!flush) mma_commit_elect(smem_addr(&bars.k_empty[gj & 1]));
        }
        if (!ok || flush) break;
        kv += nB;
      }
      // every MMA issued above has completed before TMEM is released
      mma_commit_elect(smem_addr(&bars.drain));
      mbar_wait_drain(smem_addr(&bars.drain), 0, p.status, p.wait_limit_ns);
      __syncwarp();
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
    // ------------------------------------------------------------------ softmax / epilogue
    // warps 4..11 tile A, 12..19 tile B; within a tile the first four warps take key columns
    // 0..63 and the next four 64..127 of the same rows (lane quarter = warp % 4)
    const int t = (warp - 4) >> 3;        // query tile
    const int half = ((warp - 4) >> 2) & 1;
    const int c0 = half * 64;             // this warp's 64 columns of S, P and O
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t bar_id = 1 + t * 4 + quarter;  // named barrier of the two warps of a row
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_off + t * 128 + c0;
    const uint32_t tO = tmem + lane_off + 256 + t * 128 + c0;
    const float sl2 = p.scale_log2;
    uint32_t scnt = 0;  // s_full phases consumed (key tiles processed) by this tile's warps
    // Both warps of a row pass the same named barriers in the same order on every path, and
    // decide together whether to go on (a wait that gave up in one of them stops both).
    for (int k = 0;; k++) {
      bool got = mbar_wait<1>(smem_addr(&bars.q_full[0]), k & 1, ab);
      __syncwarp();
      got = __all_sync(0xffffffffu, got);
      const int item = got ? item_slot[k & 1] : -1;
      __syncwarp();
      if (item >= 0 && lane == 0) mbar_arrive(smem_addr(&bars.q_empty[0]));  // id taken
      if (!named_bar_and(bar_id, 64, item >= 0)) break;
      const FwdItem it = decode_item(p, item);
      const int qt = it.qt0 + t;
      const int n = t ? it.nB : it.nA;
      float m = -INFINITY, l = 0.f;   // running max (shared by both halves) and partial sum
      bool ok = true;
      for (int j = 0; j < n; j++, scnt++) {
        ok = mbar_wait<1>(smem_addr(&bars.s_full[t]), scnt & 1, ab);
        __syncwarp();
        ok = __all_sync(0xffffffffu, ok);
        tc_fence_after();
        const bool diag = p.causal && j == qt;
        float mraw = -INFINITY, rs = 0.f, alpha = 1.f;
        bool rescale = false, stored = false;
        if (ok) {
          uint32_t x0[32], x1[32];
          load_s64(tS, diag, c0, row, x0, x1);
          mraw = max64(x0, x1);
          // Fast path: this warp's half rows all have a running max m already (m is -inf
          // only before the first key tile) and stay within 2^8 of it, so P = exp2(S sl2 -
          // m) can be written at once, before the other half's max is known. A half row
          // that is wholly masked (mraw = -inf) gets P = 0 here. The decision is per warp:
          // the TMEM stores are warp-collective.
          if (__all_sync(0xffffffffu, m > -INFINITY && mraw * sl2 <= m + kRescaleThreshold)) {
            rs = write_p64(x0, x1, sl2, -m, tS);
            stored = true;
          }
        }
        // Slow path, taken by both warps of the row together when either half has not
        // written its P (first key tile, a max that grew past the threshold) or gave up
        // waiting: exchange the exact max; m moves to ceil(max * sl2), an integer, so a P
        // already written with the old m is brought to the new one by an exact power of two.
        if (named_bar_or(bar_id, 64, !stored || !ok)) {
          xmax[scnt & 1][t][half][row] = mraw;
          ok = named_bar_and(bar_id, 64, ok);
          if (!ok) break;
          const float mt = fmaxf(mraw, xmax[scnt & 1][t][half ^ 1][row]) * sl2;
          const float mnew = mt > m + kRescaleThreshold ? ceilf(mt) : m;
          alpha = exp2_int(m - mnew);  // 0 while m is -inf, 1 if m stays
          rescale = j > 0 && mnew != m;
          if (!stored) {  // (warp-uniform) S is intact: nothing was written over it
            uint32_t x0[32], x1[32];
            load_s64(tS, diag, c0, row, x0, x1);
            rs = write_p64(x0, x1, sl2, -mnew, tS);
          } else if (__any_sync(0xffffffffu, mnew != m)) {
            scale_p64(tS, alpha);
            rs *= alpha;
          }
          m = mnew;
        }
        l = l * alpha + rs;
        // O rescale of this warp's 64 columns; PV of the previous key tile has completed
        // (S_t(j) landed after it), and PV of this one waits for p_full below
        if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
          for (int ch = 0; ch < 4; ch++) {
            uint32_t o[16];
            tmem_ld16(tO + ch * 16, o);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 16; c++) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
            tmem_st16(tO + ch * 16, o);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(smem_addr(&bars.p_full[t]));
      }
      if (ok) {
        ok = mbar_wait<1>(smem_addr(&bars.o_final[t]), k & 1, ab);
        __syncwarp();
        ok = __all_sync(0xffffffffu, ok);
      }
      // total row sum = both halves' partial sums; the second barrier also settles whether
      // both warps go on
      if (half == 1) xsum[t][row] = l;
      named_bar_sync(bar_id, 64);
      if (half == 0) xsum[t][row] += l;
      ok = named_bar_and(bar_id, 64, ok);
      const float ltot = xsum[t][row];
      if (!ok) break;
      tc_fence_after();
      const float inv_l = 1.f / ltot;
      uint32_t w[32];  // the row's 64 outputs, bf16 pairs; 16-byte chunk c is w[4c .. 4c + 3]
#pragma unroll
      for (int ch = 0; ch < 2; ch++) {
        uint32_t o[32];
        tmem_ld32(tO + ch * 32, o);
        tmem_wait_ld();
#pragma unroll
        for (int c2 = 0; c2 < 16; c2++)
          w[ch * 16 + c2] = pack_bf16x2(__uint_as_float(o[2 * c2]) * inv_l,
                                        __uint_as_float(o[2 * c2 + 1]) * inv_l);
      }
      // each store below then writes four whole 128-byte row segments, where a store of
      // the row a lane holds would write 16 bytes to each of 32 rows
      transpose_chunks8(w, lane);
      // the tile's rows are consecutive tokens from m0 (a 128-row tile never straddles the
      // wrap of the roll, G / 2 being a multiple of 128)
      const int m0 = src_row(it.r0 + t * kTile, it.sh, p.G, p.N);
      const size_t rstride = (size_t)p.Hq * kD;
      __nv_bfloat16* obase = static_cast<__nv_bfloat16*>(p.o) +
                             ((size_t)(it.b * p.N + m0 + quarter * 32 + (lane & ~7)) * p.Hq +
                              it.h) * kD + c0 + (lane & 7) * 8;
#pragma unroll
      for (int c = 0; c < 8; c++)
        *reinterpret_cast<uint4*>(obase + c * rstride) =
            make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
      if (half == 0)
        p.lse[((size_t)it.b * p.Hq + it.h) * p.N + m0 + row] =
            (m + __log2f(ltot)) * 0.69314718055994531f;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

cudaError_t launch_tc_fwd(const Params& p, cudaStream_t st) {
  CUtensorMap tq, tk, tv;
  cudaError_t e;
  if ((e = make_tmap_bf16_2d(&tq, p.qr, kD, (uint64_t)p.B * p.Hq * p.N, kD * 2, 64, kTile)))
    return e;
  if ((e = make_tmap_bf16_2d(&tk, p.kr, kD, (uint64_t)p.B * p.Hkv * p.N, kD * 2, 64, kTile)))
    return e;
  if ((e = make_tmap_bf16_3d(&tv, p.v, kD, p.Hkv, (uint64_t)p.B * p.N, kD * 2,
                             (uint64_t)p.Hkv * kD * 2, 64, kTile)))
    return e;
  if ((e = cudaFuncSetAttribute(tc_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)kSmemBytes)))
    return e;
  // setmaxnreg.inc waits until the registers it asks for are free: refuse to launch unless the
  // split fits what the launch hands out
  cudaFuncAttributes fa;
  if ((e = cudaFuncGetAttributes(&fa, tc_fwd_kernel))) return e;
  if (128 * kRegsOther + (kThreads - 128) * kRegsSoftmax > kThreads * fa.numRegs)
    return cudaErrorInvalidConfiguration;
  // persistent: at most one CTA per SM (one fits), each taking items until none is left
  const long items = (long)p.B * p.Hq * (p.N / p.G) * (p.G / kTile / 2);
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev))) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev))) return e;
  const unsigned grid = (unsigned)(items < sms ? items : sms);
  tc_fwd_kernel<<<dim3(grid), dim3(kThreads), kSmemBytes, st>>>(p, tq, tk, tv, (int)items);
  return cudaGetLastError();
}

}  // namespace s2
