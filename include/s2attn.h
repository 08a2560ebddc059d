/*
 * s2attn.h - C ABI of libs2attn.so: shifted sparse attention (S2-Attn) forward and backward
 * on one NVIDIA B200 (sm_100a), with RoPE and linear position interpolation fused in.
 *
 * The operation (sources are web pages on LongLoRA, cited by title and section):
 *  - RoPE with position interpolation ("LoRA for Long-Context Adaptation", sections
 *    "Why vanilla LoRA under-delivers on long context" and "Position interpolation: the
 *    prerequisite"): channel pair (2i, 2i+1) of q and of k at token m (0-based, original
 *    order) is rotated by phi = (m / pi_scale) * rope_base^(-2i/d). v is not rotated.
 *  - Half-group shift ("LongLoRA and Shifted Sparse Attention (S^2-Attn)", definition;
 *    "LongLoRA: Efficient 100k Context LLM Fine-Tuning Guide", "How Shifted Short Attention
 *    Works" and "Implementation ... Step 1"): query heads h >= H_q/2 (and kv heads
 *    >= H_kv/2) see the sequence rolled by -G/2 with wrap-around: rolled row r holds
 *    original token (r + G/2) mod N. Two other head patterns are selectable through the
 *    mode argument (S2_SHIFT_* below).
 *  - Group fold: rolled rows are cut into N/G groups of G rows; inside each group,
 *    softmax(q k^T / sqrt(d)) v with a causal mask on group-local positions (no mask
 *    without S2_CAUSAL). GQA: query head h uses kv head h / (H_q / H_kv).
 *  - Roll back: each shifted head's output row r is stored at token (r + G/2) mod N.
 *  - Backward: gradients of the above with respect to the pre-RoPE q, k and to v; dk and
 *    dv of a kv head are summed over the query heads that share it.
 *
 * Layouts (all dense, row-major, element = dtype unless noted):
 *    q, o, dout, dq : [B][N][H_q][d]      k, v, dk, dv : [B][N][H_kv][d]
 *    lse            : [B][H_q][N] float32, natural log of the softmax normaliser of the
 *                     scaled scores, in original token order.
 * Every pointer argument is a DEVICE pointer (cudaMalloc'd or equivalent), 16-byte aligned.
 * The caller owns every buffer, including the workspace; the library allocates no device
 * memory in these calls. All work is enqueued on cuda_stream (a cudaStream_t; NULL = the
 * legacy default stream) and runs asynchronously; no call synchronises.
 * Outputs are overwritten, never accumulated into.
 *
 * Errors: argument errors are returned before anything is enqueued and leave the outputs
 * untouched. A failed CUDA launch or query returns S2_ERR_CUDA. Device-side bounded waits
 * that expire set a status word in the workspace; s2attn_device_status() reads it.
 * No C++ exception crosses this interface. All functions are thread-safe.
 */
#ifndef S2ATTN_H
#define S2ATTN_H

#include <stddef.h>

#if defined(__GNUC__)
#define S2_API __attribute__((visibility("default")))
#else
#define S2_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  S2_OK = 0,
  S2_ERR_NULL = 1,           /* a required pointer is NULL */
  S2_ERR_SHAPE = 2,          /* B, N, H_q, H_kv, G <= 0; G > N; N % G != 0; G odd;
                                H_q or H_kv odd; H_q % H_kv != 0 */
  S2_ERR_DTYPE = 3,          /* dtype is not an s2_dtype value */
  S2_ERR_HEADDIM = 4,        /* d is not a multiple of 32 in [32, 256] */
  S2_ERR_ALIGN = 5,          /* a pointer is not 16-byte aligned */
  S2_ERR_WORKSPACE = 6,      /* workspace NULL or ws_bytes < s2attn_workspace_bytes(...) */
  S2_ERR_CUDA = 7,           /* a CUDA runtime/driver call failed */
  S2_ERR_DEVICE_TIMEOUT = 8, /* a bounded device-side wait expired (see s2attn_device_status) */
  S2_ERR_ARG = 9,            /* pi_scale or rope_base not finite and > 0, or a bad mode */
  S2_ERR_STALE_WORKSPACE = 10 /* (device status) s2attn_bwd_after_fwd was given a workspace
                                 whose rotation came from another forward */
} s2_status;

/* The `mode` argument of the attention calls: S2_CAUSAL or 0, ORed with one S2_SHIFT_*
 * pattern. The values 0 and 1 are the plain causal flag with the method's half-head shift.
 * Any other bit set is rejected with S2_ERR_ARG. Query heads follow their kv head under
 * every pattern; with H_kv even, "h >= H_q/2" and "h / (H_q/H_kv) >= H_kv/2" agree. */
#define S2_CAUSAL 0x01          /* causal mask on group-local positions; absent: no mask,
                                   every query sees its whole group (the full-group reading
                                   of "LoRA for Long-Context Adaptation", "Shifted sparse
                                   attention: making training feasible") */
#define S2_SHIFT_HALF 0x00      /* the second half of the heads is shifted (the definition) */
#define S2_SHIFT_ALTERNATE 0x10 /* every odd kv head is shifted: the alternate-heads
                                   wording of the same section of "LoRA for Long-Context
                                   Adaptation" */
#define S2_SHIFT_NONE 0x20      /* no head is shifted. With G == N and S2_CAUSAL this is
                                   plain dense causal attention: the inference mode of the
                                   guide's "Dual-Mode" paragraph ("LongLoRA: Efficient 100k
                                   Context LLM Fine-Tuning Guide") */

typedef enum {
  S2_BF16 = 0, /* bfloat16 storage, fp32 accumulation, tensor cores where the shape allows */
  S2_FP32 = 1  /* float32 storage and arithmetic (CUDA cores) */
} s2_dtype;

/* Bytes of device workspace that s2attn_fwd / s2attn_bwd need for this shape (it does not
 * depend on G or mode). Returns 0 for arguments that s2attn_fwd would reject with
 * S2_ERR_SHAPE, S2_ERR_HEADDIM or S2_ERR_DTYPE. The workspace holds the rotated q and k
 * (head-major, original token order), the RoPE cos/sin table, the backward's row sums
 * D = rowsum(dO * O) and per-row terms (-LSE and -D as bf16 parts, 32 bytes per query
 * row), the device status word, the fingerprint of the rotation and the work counters of
 * the persistent kernels. A workspace serves one call at a time: calls whose kernels may overlap on the
 * GPU (e.g. on two streams) need a workspace each. */
S2_API size_t s2attn_workspace_bytes(int B, int N, int H_q, int H_kv, int d, int dtype);

/* Forward: o and lse from q, k, v. See the header comment for the operation and layouts.
 * G: group size (even, divides N). mode: S2_CAUSAL (causal mask inside each group) or 0,
 * ORed with the shifted-head pattern (S2_SHIFT_HALF = 0 by default).
 * pi_scale: position interpolation factor s = L_new / L_orig (1 = plain RoPE).
 * rope_base: RoPE base (10000 for LLaMA2). Base scaling, the other rescaling of the same
 * pages ("LoRA for Long-Context Adaptation", "A training recipe", step 1), is
 * pi_scale = 1 with rope_base multiplied by the extension ratio. */
S2_API s2_status s2attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                     int B, int N, int H_q, int H_kv, int d, int G, int mode,
                     float pi_scale, float rope_base, int dtype,
                     void* workspace, size_t ws_bytes, void* cuda_stream);

/* Backward: dq, dk, dv from q, k, v, the forward's o and lse, and dout = dL/do.
 * Same shape arguments as the forward; o and lse must come from s2attn_fwd with the same
 * arguments. The workspace may be the forward's or another one of the same size. */
S2_API s2_status s2attn_bwd(const void* q, const void* k, const void* v, const void* o,
                     const float* lse, const void* dout, void* dq, void* dk, void* dv,
                     int B, int N, int H_q, int H_kv, int d, int G, int mode,
                     float pi_scale, float rope_base, int dtype,
                     void* workspace, size_t ws_bytes, void* cuda_stream);

/* Backward that reuses the forward's rotation: identical arguments, semantics and outputs
 * to s2attn_bwd, but it skips the RoPE + PI pass (one read of q, k and one write of the
 * rotated q~, k~ and of the (cos, sin) table) and reads those from the workspace instead.
 * Precondition: `workspace` is the one s2attn_fwd used for these same q, k and
 * shape/G/mode/pi_scale/rope_base/dtype arguments, and neither it (beyond the status word)
 * nor q, k changed since. The forward records a fingerprint of those arguments (with the q
 * and k pointers) in the workspace; this call compares it on the device and, on a mismatch,
 * leaves S2_ERR_STALE_WORKSPACE for s2attn_device_status() and its gradients are undefined
 * (the tensor-core kernels skip their work). New contents written into the same q, k
 * buffers are not detected. This is the training-loop order (forward, then backward of the same
 * batch); the method is unchanged, the rotation is computed once per step instead of twice
 * ("LongLoRA: Efficient 100k Context LLM Fine-Tuning Guide", Step 1 applies RoPE once). The
 * status word is reset at the start, as in every other call. */
S2_API s2_status s2attn_bwd_after_fwd(const void* q, const void* k, const void* v,
                                      const void* o, const float* lse, const void* dout,
                                      void* dq, void* dk, void* dv, int B, int N, int H_q,
                                      int H_kv, int d, int G, int mode, float pi_scale,
                                      float rope_base, int dtype, void* workspace,
                                      size_t ws_bytes, void* cuda_stream);

/* Bytes of the fixed scratch array that s2attn_fwd_noalloc uses on each device. */
#define S2ATTN_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)

/* Forward for callers that cannot allocate device memory per call (a plugin whose host
 * application owns every device allocation, a latency-critical loop that cannot afford
 * cudaMalloc's implicit synchronisation, a C caller with no allocator). The pages have no
 * counterpart: this is a deployment variant of s2attn_fwd, not part of the method.
 * Same arguments, semantics and outputs as s2attn_fwd, minus the workspace: the scratch is
 * a fixed S2ATTN_NOALLOC_SCRATCH_BYTES array inside the library, which every device that
 * loads the library holds until the process exits. Neither this call nor the library
 * allocates memory (no cudaMalloc, cudaFree or allocating library routine).
 *  - Limit: shapes whose s2attn_workspace_bytes() exceeds S2ATTN_NOALLOC_SCRATCH_BYTES are
 *    rejected with S2_ERR_WORKSPACE before anything is enqueued.
 *  - Set-up: the first call on a device looks up the array's device address (with that
 *    device current) and caches it, keyed by the device's CUDA context, so that after a
 *    device reset (a new context) the address is looked up again; make the first call,
 *    and the first call after a reset, before any stream capture.
 *  - Sharing: every call on a device uses the same array and leaves its contents behind
 *    (each call rewrites what it reads, and resets the status word first). Calls whose
 *    kernels overlap on the GPU (e.g. on two streams) race on the array: serialise them. */
S2_API s2_status s2attn_fwd_noalloc(const void* q, const void* k, const void* v, void* o,
                                    float* lse, int B, int N, int H_q, int H_kv, int d, int G,
                                    int mode, float pi_scale, float rope_base, int dtype,
                                    void* cuda_stream);

/* Device status of s2attn_fwd_noalloc, for the same callers (no passage of the pages
 * corresponds to it). Their status word lives in the library's fixed scratch array, which
 * they cannot address, so s2attn_device_status() cannot reach it. This call waits for
 * cuda_stream, then reads and clears the status word of the current device's scratch:
 * S2_OK, or S2_ERR_DEVICE_TIMEOUT if a bounded wait of the last no-allocation forward on
 * this device expired (its o and lse are then undefined). S2_ERR_CUDA on a CUDA error.
 * It allocates nothing. Every no-allocation call on a device shares this word, so read it
 * after the call whose status is wanted and before the next one starts. */
S2_API s2_status s2attn_noalloc_device_status(void* cuda_stream);

/* Which kernel family s2attn_fwd and s2attn_bwd launch for these arguments:
 * 1 = tcgen05 tensor-core kernels (bf16, d == 128, G % 256 == 0),
 * 0 = CUDA-core kernels (any other valid shape, and every fp32 call), -1 = invalid. */
S2_API int s2attn_kernel_path(int B, int N, int H_q, int H_kv, int d, int G, int mode, int dtype);

/* Waits for cuda_stream, then reads and clears the device status word of the workspace
 * used by the last call on it: S2_OK, S2_ERR_DEVICE_TIMEOUT if a bounded wait in a kernel
 * expired (that kernel's outputs are then undefined), or S2_ERR_STALE_WORKSPACE if
 * s2attn_bwd_after_fwd found another forward's rotation there (its gradients were not
 * computed). S2_ERR_CUDA on a CUDA error. */
S2_API s2_status s2attn_device_status(void* workspace, size_t ws_bytes, void* cuda_stream);

/* Self-test of the device-side failure path: enqueues one tiny kernel whose bounded wait
 * on an mbarrier (which nothing ever arrives on) expires after 50 ms and records the
 * timeout in the workspace's status word, exactly as an expired wait in the attention
 * kernels does. Afterwards s2attn_device_status() must report S2_ERR_DEVICE_TIMEOUT and
 * the CUDA context stays usable. Needs only the first 256 bytes of a workspace. */
S2_API s2_status s2attn_selftest_wait_timeout(void* workspace, size_t ws_bytes,
                                              void* cuda_stream);

/* Self-test of the tensor-core kernels' own failure path. Runs the tcgen05 forward
 * (site S2_INJECT_FWD; the arguments of s2attn_fwd, dout/dq/dk/dv unused and may be NULL)
 * or the whole backward (site S2_INJECT_DKDV; the arguments of s2attn_bwd, with o and lse
 * from a forward of the same inputs) with
 * two changes: every bounded wait gives up after 50 ms instead of 2 s, and the MMA issuer of
 * the launch's first CTA withholds one barrier arrival (the completion of one score tile:
 * tile B at key tile 1 of its first item in the forward, S^T of pair 1 of key tile 0 in the
 * dK/dV pass). The waits on it expire, the CTA records S2_ERR_DEVICE_TIMEOUT in the status
 * word, every CTA of the launch gives up, drains its TMA loads and MMAs and frees its TMEM;
 * the CUDA context stays usable. Afterwards s2attn_device_status() reports the timeout and
 * the outputs are undefined. Needs the tcgen05 path (s2attn_kernel_path() == 1), else
 * S2_ERR_ARG; argument checks as in s2attn_fwd / s2attn_bwd. No trap, fault or endless
 * wait is involved: the failure is a missing arrival and every wait is bounded. */
#define S2_INJECT_FWD 1
#define S2_INJECT_DKDV 2
S2_API s2_status s2attn_selftest_inject(int site, const void* q, const void* k, const void* v,
                                        void* o, float* lse, const void* dout, void* dq,
                                        void* dk, void* dv, int B, int N, int H_q, int H_kv,
                                        int d, int G, int mode, float pi_scale,
                                        float rope_base, int dtype, void* workspace,
                                        size_t ws_bytes, void* cuda_stream);

/* Self-test of the FMA-pipe exp2 the softmax kernels use for part of their exponentials
 * (range reduction + degree-3 polynomial): y[i] = 2^x[i] for n device floats, enqueued on
 * cuda_stream. Accurate to a relative 1e-4 for x in [-125, 127]. */
S2_API s2_status s2attn_selftest_exp2(const float* x, float* y, int n, void* cuda_stream);

/* Static, NUL-terminated description of a status code. */
S2_API const char* s2attn_status_string(int status);

/* Kernel timing for measurement. When enabled, every kernel the library launches is
 * bracketed by two CUDA events recorded on its launching stream (a bounded pool; records
 * beyond it are dropped and counted). s2attn_profile_query() waits for those events and
 * returns per-kernel launch counts and summed durations. */
S2_API s2_status s2attn_profile_enable(int on);  /* on = 1 starts afresh, 0 stops recording */
S2_API int s2attn_profile_num_kernels(void);     /* number of kernel ids */
S2_API s2_status s2attn_profile_query(int kernel_id, const char** name, int* launches,
                               double* total_ms);
S2_API int s2attn_profile_dropped(void);         /* records dropped since the last enable */

#ifdef __cplusplus
}
#endif

#endif /* S2ATTN_H */
