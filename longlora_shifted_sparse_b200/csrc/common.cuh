// Shared definitions of the S2-Attn CUDA library: argument block, index maps, conversions.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace s2 {

// Everything a kernel of one call needs. Built once per call on the host, passed by value.
struct Params {
  int B, N, Hq, Hkv, d, G, causal;
  int shift;         // ShiftPattern: which heads are rolled by -G/2
  float pi_scale, rope_base;
  float scale;       // 1 / sqrt(d)
  float scale_log2;  // log2(e) / sqrt(d): scores go straight to the exp2 domain
  // caller tensors
  const void* q;
  const void* k;
  const void* v;
  void* o;
  float* lse;
  const void* dout;
  void* dq;
  void* dk;
  void* dv;
  // workspace views
  void* qr;         // rotated q, [B][Hq][N][d], original token order
  void* kr;         // rotated k, [B][Hkv][N][d], original token order
  float2* cs;       // (cos, sin) of (m / s) * theta_i, [N][d/2]
  float* Dsum;      // rowsum(dO * O), [B][Hq][N]
  // per query row, the backward's row terms as a 16-element bf16 row [B][Hq][N][16]:
  // -LSE*sqrt(d) split into three bf16 parts (elements 0..2), -D into two (3, 4), zeros.
  // The tensor-core dK/dV pass adds them to S^T and dP^T as one more MMA k-step.
  void* rowterms;
  unsigned* status; // device status word (bit 0: a bounded wait expired)
  // failure-path testing: the time limit of every bounded wait, and which kernel (if any)
  // withholds one barrier arrival so that a wait expires (InjectSite; 0 in normal calls)
  unsigned long long wait_limit_ns;
  int inject;
  // hash of the call's arguments that determine the rotation held in the workspace (shape,
  // mode, pi_scale, rope_base, dtype, the q and k pointers): a call that rotates stores it
  // in the status block; a backward that reuses the rotation compares it (check_fingerprint)
  unsigned long long fingerprint;
  int check_fingerprint;
};

// Where a failure-path self-test withholds one arrival (the issuer of CTA 0 skips the
// commit that would complete a score tile): kInjectFwd in the forward (score tile A, key
// tile 1 of its first item), kInjectDkdv in the dK/dV pass (S^T of pair 1).
enum InjectSite : int { kInjectNone = 0, kInjectFwd = 1, kInjectDkdv = 2 };

// Status word bits: a bounded wait expired; a backward that reuses the forward's rotation
// found a workspace whose last rotation came from other arguments (its kernels then skip).
enum StatusBits : unsigned { kStatusTimeout = 1u, kStatusStale = 2u };
// Words 8 and 9 of the workspace's 256-byte status block: the fingerprint of the rotation.
constexpr int kFingerprintWord = 8;
// Time limit of one bounded wait in a normal call (2 s: far beyond any wait of a working
// kernel, short enough that a stuck launch ends with an error instead of hanging).
constexpr unsigned long long kWaitLimitNs = 2000000000ull;
// The same limit in the failure-path self-tests, which make a wait expire on purpose.
constexpr unsigned long long kSelftestWaitLimitNs = 50000000ull;
// Words after the status word (same 256-byte block of the workspace): the work-item
// counters of the persistent kernels. The RoPE pass zeroes them all at the start of every
// forward, the row-sum pass at the start of every backward.
constexpr int kFwdWorkCounter = 1;
constexpr int kDqWorkCounter = 2;
constexpr int kNumWorkCounters = 2;

// Which heads are rolled by -G/2. kShiftHalf: the second half of the heads (the method's
// definition). kShiftAlternate: every odd kv head (the alternate-heads wording of the
// pages' group figure). kShiftNone: no head (with G = N, dense causal attention).
enum ShiftPattern : int { kShiftHalf = 0, kShiftAlternate = 1, kShiftNone = 2 };

// A query head is shifted with its kv head (h -> h / (Hq/Hkv)). With Hkv even this is the
// same as "h >= Hq/2" for the half pattern.
__host__ __device__ inline bool kv_head_shifted(int kvh, const Params& p) {
  if (p.shift == kShiftAlternate) return (kvh & 1) != 0;
  if (p.shift == kShiftNone) return false;
  return kvh >= p.Hkv / 2;
}
__host__ __device__ inline bool q_head_shifted(int h, const Params& p) {
  return kv_head_shifted(h / (p.Hq / p.Hkv), p);
}

// Work order of the tensor-core kernels: CTA x of a grid of U units (b, kv head, group)
// times W items per unit -> (unit, item), item 0 being a unit's heaviest item. Units are
// taken `chunk` at a time (kLptChunk unless the kernel sizes it); inside a chunk the items
// run heaviest first across all of the chunk's units. The last wave then holds only light
// items (longest-processing-time order, a short tail), while the few units in flight keep the
// tiles they share resident in L2.
constexpr int kLptChunk = 8;
__device__ inline void chunked_lpt(int x, int U, int W, int& unit, int& item,
                                   int chunk = kLptChunk) {
  const int c0 = x / (chunk * W) * chunk;
  const int cc = min(chunk, U - c0);
  const int r = x - c0 * W;
  item = r / cc;
  unit = c0 + (r - item * cc);
}

// Rolled row r -> original token. Rolling by -G/2 puts token (r + G/2) mod N at row r.
__host__ __device__ inline int src_row(int r, bool shifted, int G, int N) {
  if (!shifted) return r;
  int m = r + G / 2;
  return m >= N ? m - N : m;
}

template <typename T> __device__ inline float to_f32(T x);
template <> __device__ inline float to_f32<float>(float x) { return x; }
template <> __device__ inline float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}

template <typename T> __device__ inline T from_f32(float x);
template <> __device__ inline float from_f32<float>(float x) { return x; }
template <> __device__ inline __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

__device__ inline float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// 8 x 8 transpose of 16-byte chunks inside each group of eight lanes of a warp. Lane 8g + i
// passes in the eight chunks of its own row (chunk c = w[4c .. 4c + 3]) and gets back chunk i
// of the group's eight rows (w[4c ..] = chunk i of row 8g + c): the eight lanes of a group
// then hold one 128-byte segment of a row together, so that a store of chunk c, or a read
// of data laid out like the row, touches whole segments. Three butterfly stages of
// shuffles; every index is static, so the array stays in registers.
__device__ __forceinline__ void transpose_chunks8(uint32_t (&w)[32], int lane) {
  const int l8 = lane & 7;
#pragma unroll
  for (int bit = 4; bit >= 1; bit >>= 1) {
    const bool up = (l8 & bit) != 0;
#pragma unroll
    for (int c = 0; c < 8; c++) {
      if (c & bit) continue;
#pragma unroll
      for (int e = 0; e < 4; e++) {
        const uint32_t mine = w[4 * c + e], other = w[4 * (c ^ bit) + e];
        const uint32_t got = __shfl_xor_sync(0xffffffffu, up ? mine : other, bit);
        if (up)
          w[4 * c + e] = got;
        else
          w[4 * (c ^ bit) + e] = got;
      }
    }
  }
}

}  // namespace s2
