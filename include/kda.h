/*
 * kda.h -- C ABI of the B200 (sm_100a) Kimi Delta Attention library.
 *
 * The operator.  The page "Kimi K3: Open Frontier Intelligence and
 * Implementation Framework" (section "Technical Architecture and Scaling
 * Efficiency", sub-section "Hybrid Attention Mechanism", KDA bullet)
 * describes Kimi Delta Attention as the delta-rule recurrence extended with
 * a channel-wise forget gate whose decay is bounded below, which lets the
 * diagonal and off-diagonal tiles of a chunked evaluation run as dense
 * tensor-core products.  Per head, with a d_k x d_v state S:
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *     o_t = S_t^T q_t,            alpha_t = exp(log_alpha_t) per channel.
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller; the
 *     library never allocates, frees or retains them.  Every tensor is dense
 *     row-major and its base address must be 16-byte aligned.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Work is enqueued asynchronously; the call returns once it is
 *     enqueued.
 *   - Host-side validation (NULL pointers, alignment, sizes, dtypes) is done
 *     before anything is enqueued and returns a kda_status synchronously;
 *     nothing runs on the device when a call returns an error.
 *   - Launch failures return KDA_ERR_CUDA.  Problems only the device can see
 *     (malformed cu_seqlens contents) are written to a status word in the
 *     workspace, read back with kda_workspace_status().
 *   - Token axis: sequences are packed back to back along a token axis of
 *     length total_tokens and delimited by cu_seqlens.
 *   - Supported shapes: Dk, Dv in {64, 128}; chunk == 64; H >= 1.
 *   - The factorisation exp(g_r - g_s) = exp(g_r) * exp(-g_s) used inside a
 *     chunk needs the in-chunk cumulative log-decay of every channel to stay
 *     above -80 (fp32 exponent range): e.g. alpha >= exp(-1.25) per token at
 *     chunk 64.  That is the lower bound on the decay the method relies on;
 *     the library does not clamp log_alpha.  The chunked kernels check it:
 *     a log_alpha above 0 or not finite, or a channel whose cumulative
 *     log-decay over one chunk falls below -80, records KDA_ERR_DECAY in the
 *     workspace status word (no trap, nothing read or written out of range).
 *     The outputs and final state of the (sequence, head) chains that hold
 *     such a chunk are then unspecified; every other chain is unaffected.
 *   - Every entry point makes the device that owns its tensors current for
 *     the launches and restores the caller's current context (device) before
 *     it returns, on success and on error.
 */
#ifndef KDA_H
#define KDA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define KDA_ABI_VERSION 4

typedef enum kda_status {
    KDA_OK = 0,
    KDA_ERR_INVALID = 1,      /* NULL pointer, non-positive size, bad value      */
    KDA_ERR_UNSUPPORTED = 2,  /* Dk/Dv/chunk/dtype combination not implemented    */
    KDA_ERR_ALIGN = 3,        /* a tensor base address is not 16-byte aligned     */
    KDA_ERR_WORKSPACE = 4,    /* workspace NULL, misaligned or too small          */
    KDA_ERR_CUDA = 5,         /* a CUDA runtime call or kernel launch failed      */
    KDA_ERR_TIMEOUT = 6,      /* a bounded device-side wait gave up               */
    KDA_ERR_SEQLENS = 7,      /* device saw cu_seqlens not 0..total_tokens monotone */
    KDA_ERR_SLOT = 8,         /* device saw a snapshot-pool slot outside the pool */
    KDA_ERR_DECAY = 9,        /* device saw a gate outside the chunked form's range */
    KDA_ERR_BOUNDS = 10       /* debug builds only: an index outside its buffer (skipped) */
} kda_status;

typedef enum kda_dtype {
    KDA_F32 = 0,
    KDA_BF16 = 1
} kda_dtype;

/* Problem description shared by kda_forward and kda_decode_step. */
typedef struct kda_params {
    int32_t num_seqs;      /* N: number of sequences (prefill) or decode rows   */
    int32_t total_tokens;  /* T_tot: packed token count (prefill); ignored by decode */
    int32_t H;             /* heads                                            */
    int32_t Dk;            /* key / query width: 64 or 128                     */
    int32_t Dv;            /* value width: 64 or 128                           */
    int32_t chunk;         /* prefill chunk length; must be 64                 */
    int32_t io_dtype;      /* kda_dtype of q, k, v and out                     */
    int32_t gate_dtype;    /* kda_dtype of log_alpha and beta                  */
    int32_t flags;         /* 0, or KDA_FLAG_* bits below                      */
} kda_params;

/* Evaluate a bf16 problem with the fp32 CUDA-core prefill instead of the
 * tensor-core one (slower; for cross-checking the two kernels). */
#define KDA_FLAG_FORCE_SIMT 1
/* Use the single-kernel tensor-core prefill even when the workspace is large
 * enough for the two-pass one (for cross-checking the two). */
#define KDA_FLAG_FUSED_TC 2
/* Failure-path check: on the two-pass path the chain pass's MMA issuer waits
 * on a barrier nothing arrives on.  The bounded wait gives up after about
 * 2 s, every role of the CTA winds down (MMAs and copies drained, tensor
 * memory freed), outputs are left incomplete and KDA_ERR_TIMEOUT is recorded
 * in the workspace status; the CUDA context stays usable.  No fault, trap or
 * unbounded wait is involved. */
#define KDA_FLAG_TEST_STALL 4

/*
 * kda_forward_workspace_size -- bytes of device workspace for the fastest
 * kda_forward path of this problem.  Returns 0 when `p` is NULL or invalid.
 * The workspace must be 256-byte aligned; its contents need no
 * initialisation and are overwritten by every call.
 *
 * Every path needs a status word and the per-sequence work order (256 bytes
 * + 4 N, rounded up to 256).  For bf16 inputs with Dk = Dv = 128 the fastest
 * path is a two-pass tensor-core prefill that also stores, per 64-token chunk
 * and head, a 65 KB operand packet: about (total_tokens / 64 + N) * H * 65 KB
 * (~1 KB per token and head).  Given less than that (but at least the
 * minimum) kda_forward runs the single-kernel tensor-core prefill instead.
 */
size_t kda_forward_workspace_size(const kda_params *p);

/*
 * kda_forward -- chunked (chunk = 64) prefill over packed sequences.
 *
 * Computes, for every sequence n in [0, N) and head h, the recurrence above
 * over tokens cu_seqlens[n] .. cu_seqlens[n+1]-1 starting from S0[n,h]
 * (zero when S0 is NULL), writing o_t for every token and the state after
 * the sequence's last token to S_final[n,h] (skipped when S_final is NULL).
 * A zero-length sequence leaves S_final[n,h] = S0[n,h].
 *
 *   q, k       [T_tot, H, Dk]  io_dtype
 *   v          [T_tot, H, Dv]  io_dtype
 *   log_alpha  [T_tot, H, Dk]  gate_dtype   (natural log of the decay, <= 0)
 *   beta       [T_tot, H]      gate_dtype   (write strength, usually in [0,1])
 *   S0         [N, H, Dk, Dv]  fp32, or NULL for a zero initial state
 *   cu_seqlens [N + 1]         int32, device; 0 = c_0 <= c_1 <= ... <= c_N = T_tot
 *   out        [T_tot, H, Dv]  io_dtype, written
 *   S_final    [N, H, Dk, Dv]  fp32, written, or NULL
 *   workspace  device scratch: ws_bytes >= kda_forward_workspace_size(p) for
 *              the fastest path, at least the minimum described above
 *
 * Aliasing: out and S_final must not overlap any input.  S_final may be the
 * same buffer as S0 (in-place continuation of a chain); any other partial
 * overlap is undefined.  Calls that share a workspace must be ordered on the
 * same stream.
 *
 * Errors: KDA_ERR_INVALID / _UNSUPPORTED / _ALIGN / _WORKSPACE from host
 * validation; KDA_ERR_CUDA if a launch fails.  If cu_seqlens is malformed
 * the kernels skip the offending sequences (no out-of-range access) and
 * record KDA_ERR_SEQLENS in the workspace status word.
 */
kda_status kda_forward(const void *q, const void *k, const void *v,
                       const void *log_alpha, const void *beta,
                       const float *S0, const int32_t *cu_seqlens,
                       void *out, float *S_final, const kda_params *p,
                       void *workspace, size_t ws_bytes, void *stream);

/*
 * kda_forward_noalloc -- kda_forward for callers that cannot allocate device
 * memory.  The KDA description has no counterpart to this; it is a
 * convenience of this library.
 *
 * Some callers cannot hand kda_forward a workspace: engines whose device
 * memory is planned once up front and that forbid allocation while serving,
 * plug-ins running inside an application that owns the allocator, or
 * latency-critical paths that cannot take cudaMalloc's implicit device
 * synchronisation.  This entry point takes the same arguments as kda_forward
 * minus the workspace and uses a fixed scratch array held by the library:
 *
 *   - the array holds a status word and KDA_NOALLOC_MAX_SEQS int32 entries;
 *     every GPU that loads the library keeps it (about 64 KB) until exit;
 *   - p->num_seqs > KDA_NOALLOC_MAX_SEQS is rejected with
 *     KDA_ERR_UNSUPPORTED before anything is enqueued;
 *   - the first call on a device looks up the array's device address (with
 *     that device current) and caches it for the CUDA context then current;
 *     a call under another context of the device (a driver-API context the
 *     caller pushed, or a primary context re-created after cudaDeviceReset)
 *     looks it up again; make the first call in a context before any stream
 *     capture;
 *   - every call shares the array and rewrites it before use; calls whose
 *     work overlaps on the GPU race on it, so order them on one stream;
 *   - it allocates nothing (no cudaMalloc, cudaFree or allocating library
 *     call) and runs exactly the kernels of kda_forward.
 *
 * Returns the same codes as kda_forward.  What only the device can see
 * (malformed cu_seqlens, a bounded wait that gave up, an out-of-range gate)
 * goes to the array's status word; read it with kda_forward_noalloc_status.
 */
#define KDA_NOALLOC_MAX_SEQS 16384
kda_status kda_forward_noalloc(const void *q, const void *k, const void *v,
                               const void *log_alpha, const void *beta,
                               const float *S0, const int32_t *cu_seqlens,
                               void *out, float *S_final, const kda_params *p,
                               void *stream);

/*
 * kda_forward_noalloc_status -- synchronise `stream`, then copy into *status
 * the device status word that the last kda_forward_noalloc call on the device
 * owning `device_ptr` (any device pointer of that call, e.g. its cu_seqlens)
 * left in the library's scratch array: KDA_OK, or the first KDA_ERR_* code
 * the device recorded.  Like kda_forward_noalloc it allocates nothing.
 * Returns KDA_ERR_INVALID for NULL arguments or a host pointer, KDA_ERR_CUDA
 * if the synchronisation or the copy fails.
 */
kda_status kda_forward_noalloc_status(const void *device_ptr, int32_t *status, void *stream);

/*
 * kda_forward_snapshots -- kda_forward that also keeps the recurrent state in
 * a paged pool for prefix caching, and may start sequences from it.
 *
 * The page "Kimi K3: Open Frontier Intelligence and Implementation Framework",
 * section "Inference Serving", bullet "KDA-Aware Prefix Caching", keeps KDA
 * recurrent states in one paged pool so that a cached prefix can be resumed
 * at 512-token boundaries.  Here a snapshot is the fp32 state of a (sequence,
 * head) chain right after token number m * every of its sequence
 * (m = 1 .. floor(len / every)), the same state a call on just that prefix
 * would return as S_final.
 *
 *   pool       [n_slots, H, Dk, Dv] fp32, device.  Snapshot m-1 of sequence
 *              n (all heads) is written to slot slot_base[n] + m - 1.
 *   slot_base  [N] int32, device: first slot of each sequence's snapshots;
 *              negative = record none for that sequence.  May be NULL when
 *              every == 0.
 *   s0_slot    [N] int32, device, or NULL: sequence n starts from the state
 *              in slot s0_slot[n] instead of S0[n] (negative = use S0[n], or
 *              zero when S0 is NULL).
 *   every      tokens between snapshots: 0 (none) or a positive multiple of
 *              the chunk (64); the page's granularity is 512.
 *
 * Slots read through s0_slot must not be written by the same call.  A slot
 * outside [0, n_slots) is skipped on the device (nothing read or written;
 * a start slot out of range starts from zero) and KDA_ERR_SLOT is recorded
 * in the workspace status word.
 *
 * Only the two-pass tensor-core prefill keeps snapshots: bf16 q/k/v and
 * gates with Dk = Dv = 128 and ws_bytes >= kda_forward_workspace_size(p).
 * Other problems return KDA_ERR_UNSUPPORTED before anything is enqueued
 * (snap == NULL, or every == 0 with s0_slot == NULL, is plain kda_forward).
 * Other arguments and errors are those of kda_forward.
 */
typedef struct kda_snapshots {
    float *pool;
    const int32_t *slot_base;
    const int32_t *s0_slot;
    int64_t n_slots;
    int32_t every;
} kda_snapshots;

kda_status kda_forward_snapshots(const void *q, const void *k, const void *v,
                                 const void *log_alpha, const void *beta,
                                 const float *S0, const int32_t *cu_seqlens,
                                 void *out, float *S_final, const kda_params *p,
                                 const kda_snapshots *snap,
                                 void *workspace, size_t ws_bytes, void *stream);

/*
 * kda_decode_step -- one recurrent token for N independent sequences.
 *
 * For every n < N (= p->num_seqs) and head h, applies one token of the
 * recurrence to S[n,h] in place and writes its output:
 *
 *   q, k, log_alpha [N, H, Dk]  (io_dtype for q/k, gate_dtype for log_alpha)
 *   v               [N, H, Dv]  io_dtype
 *   beta            [N, H]      gate_dtype
 *   S               [N, H, Dk, Dv] fp32, read and overwritten
 *   out             [N, H, Dv]  io_dtype, written
 *
 * p->total_tokens and p->chunk are ignored.  S must not overlap any other
 * argument.  The state of each (n, h) is read once and written once per call.
 */
kda_status kda_decode_step(const void *q, const void *k, const void *v,
                           const void *log_alpha, const void *beta, float *S,
                           void *out, const kda_params *p, void *stream);

/*
 * kda_decode_multi -- n_tokens consecutive recurrent tokens per sequence in
 * one pass over the state, keeping the state after every token: the verify
 * step of speculative decoding, which accepts a prefix of draft tokens and
 * resumes from the state after the last accepted one.  (The page "Kimi K3:
 * Open Frontier Intelligence and Implementation Framework", section
 * "Inference Serving", serves K3 with an EAGLE-3-style draft model.)
 *
 *   q, k, log_alpha [N, n_tokens, H, Dk]  (io_dtype for q/k, gate_dtype)
 *   v               [N, n_tokens, H, Dv]  io_dtype
 *   beta            [N, n_tokens, H]      gate_dtype
 *   S               [N, H, Dk, Dv] fp32, read only (read once)
 *   S_tokens        [N, n_tokens, H, Dk, Dv] fp32, written: S_tokens[n, t]
 *                   is the state after token t of sequence n
 *   out             [N, n_tokens, H, Dv] io_dtype, written
 *
 * Every token applies exactly the arithmetic of kda_decode_step, so the
 * outputs and S_tokens[n, t] equal those of t + 1 successive single steps.
 * S_tokens must not overlap S.  p->total_tokens and p->chunk are ignored.
 * Errors: as kda_decode_step; n_tokens < 1 is KDA_ERR_INVALID.
 */
kda_status kda_decode_multi(const void *q, const void *k, const void *v,
                            const void *log_alpha, const void *beta, const float *S,
                            float *S_tokens, void *out, const kda_params *p,
                            int32_t n_tokens, void *stream);

/*
 * kda_backward_workspace_size -- bytes of device workspace kda_backward needs
 * for this problem; 0 when `p` is NULL or invalid.  Must be 256-byte
 * aligned; needs no initialisation.  About
 * 2 (total_tokens / 64 + N) * H * Dk * Dv * 4 bytes of states (one every 32
 * tokens), N * H * (Dv / 32) * (32 * Dk * 32 + 1024) * 4 bytes of per-CTA
 * scratch and (Dv / 32) * total_tokens * H * (3 Dk + 1) * 4 bytes of
 * per-slice partial sums.
 */
size_t kda_backward_workspace_size(const kda_params *p);

/*
 * kda_backward -- gradients of a scalar loss L through kda_forward's
 * recurrence (page "Kimi K3: Open Frontier Intelligence and Implementation
 * Framework", section "Hybrid Attention Mechanism", KDA bullet; the same
 * page trains the model built on it).  Given dL/d out and optionally
 * dL/dS_final it writes dL/d of every input:
 *
 *   q, k, v, log_alpha, beta, S0, cu_seqlens   as kda_forward (S0 may be NULL)
 *   d_out      [T_tot, H, Dv]  io_dtype, dL/d out
 *   dS_final   [N, H, Dk, Dv]  fp32, dL/dS_final, or NULL (zero)
 *   dq, dk     [T_tot, H, Dk]  fp32, written
 *   dv         [T_tot, H, Dv]  fp32, written
 *   dlog_alpha [T_tot, H, Dk]  fp32, written (gradient w.r.t. log_alpha)
 *   dbeta      [T_tot, H]      fp32, written
 *   dS0        [N, H, Dk, Dv]  fp32, written, or NULL (not computed); the
 *              gradient w.r.t. the initial state also when S0 is NULL
 *   workspace  ws_bytes >= kda_backward_workspace_size(p), 256-byte aligned
 *
 * All gradients are fp32 whatever io_dtype and gate_dtype; the arithmetic is
 * fp32 on CUDA cores.  dq, dk, dlog_alpha and dbeta are sums over the 32-wide
 * value slices: each slice's partial sum goes to the workspace and a second
 * kernel adds them in slice order, so repeated calls on the same inputs give
 * bitwise identical gradients (no atomics anywhere).  The states are
 * recomputed (the forward runs twice: once to keep the state every 32
 * tokens, once per 32 tokens in reverse order),
 * so no state from kda_forward is needed.  The recurrence is evaluated token by
 * token here, so the lower bound on the in-chunk decay stated at the top of
 * this file does not apply to this entry point.  `flags` is ignored.  Outputs may
 * not overlap inputs or each other.  Errors as kda_forward: host validation
 * codes, KDA_ERR_CUDA if a launch fails, KDA_ERR_SEQLENS recorded in the
 * workspace status word for malformed cu_seqlens (the gradients are then
 * unspecified; nothing is read or written out of range).
 */
kda_status kda_backward(const void *q, const void *k, const void *v,
                        const void *log_alpha, const void *beta,
                        const float *S0, const int32_t *cu_seqlens,
                        const void *d_out, const float *dS_final,
                        float *dq, float *dk, float *dv, float *dlog_alpha,
                        float *dbeta, float *dS0, const kda_params *p,
                        void *workspace, size_t ws_bytes, void *stream);

/*
 * kda_workspace_status -- synchronise `stream`, then copy the device status
 * word of a kda_forward workspace into *status (KDA_OK when the last call
 * that used this workspace saw nothing wrong).  Returns KDA_ERR_INVALID for
 * NULL arguments and KDA_ERR_CUDA if the copy fails.
 */
kda_status kda_workspace_status(const void *workspace, int32_t *status, void *stream);

/* Human-readable name of a status code (static storage, never NULL). */
const char *kda_status_string(kda_status s);

/* KDA_ABI_VERSION of the loaded library. */
int32_t kda_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H */
