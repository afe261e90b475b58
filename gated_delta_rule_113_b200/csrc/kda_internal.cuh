// kda_internal.cuh -- shared declarations of the KDA CUDA library (not public).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kda.h"

namespace kda {

constexpr int kChunk = 64;          // tokens per chunk of the prefill
constexpr size_t kWsHeader = 256;   // bytes: status word + padding
constexpr int kSortMax = 4096;      // sequences ordered longest-first up to this N

// Everything a prefill launch needs, already validated on the host.
struct ForwardArgs {
    const void *q, *k, *v, *log_alpha, *beta;
    const float *S0;
    const int32_t *cu_seqlens;
    void *out;
    float *S_final;
    int N, T, H, Dk, Dv;
    int io_dtype, gate_dtype;
    int32_t *status;   // device status word (workspace)
    int32_t *work_ctr; // device item counter of the key-side pass (workspace header)
    int32_t *order;    // device work order [N] (workspace)
    int32_t *chunk_off;    // device [N+1] exclusive prefix of per-sequence chunk counts, or null
    unsigned char *packets;  // device per-(chunk, head) key-side operand packets, or null
    size_t packet_slots;     // number of packets the workspace holds
    // state snapshots (two-pass path only): pool [n_slots, H, Dk, Dv] fp32
    float *snap_pool;
    const int32_t *snap_base;   // [N] first slot per sequence, negative: none
    const int32_t *s0_slot;     // [N] start slot per sequence, negative: S0; or null
    long long snap_slots;
    int snap_every_chunks;      // 0: no snapshots
    float *ckpt;                // two-pass path: state entering every chunk [slots, Dk, Dv], or null
    bool test_stall;            // chain pass waits on a barrier nobody arrives on
};

struct DecodeArgs {
    const void *q, *k, *v, *log_alpha, *beta;
    float *S;          // read; written in place when S_tokens is null
    float *S_tokens;   // [N, n_tokens, H, Dk, Dv] state after every token, or null
    int n_tokens;      // consecutive tokens per sequence (1 for a plain step)
    void *out;
    int N, H, Dk, Dv;
    int io_dtype, gate_dtype;
};

// Gradients (kda_backward), already validated on the host.
struct BackwardArgs {
    const void *q, *k, *v, *log_alpha, *beta, *d_out;
    const float *S0, *dS_final;       // either may be null
    const int32_t *cu_seqlens;
    float *dq, *dk, *dv, *dla, *dbeta;
    float *dS0;                       // or null
    int N, T, H, Dk, Dv;
    int io_dtype, gate_dtype;
    int32_t *status, *order, *chunk_off;   // workspace, as the forward's
    float *ckpt;                      // [ckpt_steps, H, Dv / 32, Dk, 32] states every kBwStep tokens
    size_t ckpt_steps;
    float *scratch;                   // per CTA: kBwStep states of a slice and kBwStep u rows
    float *part;                      // per 32-wide value slice: partial dq, dk, dla, dbeta
    size_t part_stride;               // floats per slice of `part`
};
// Floats of one value slice's partial row sums: dq, dk, dlog_alpha [T, H, Dk]
// and dbeta [T, H], padded to a multiple of 64 floats (256 bytes).
inline size_t backward_part_floats(int64_t T, int64_t H, int Dk) {
    const size_t n = (size_t)T * H * (3 * (size_t)Dk + 1);
    return (n + 63) / 64 * 64;
}
// The backward keeps the state every kBwStep tokens (two per chunk); one CTA
// (sequence, head, 32-wide value slice) recomputes kBwStep states at a time.
constexpr int kBwStep = 32;
inline size_t backward_scratch_floats(int Dk) { return (size_t)kBwStep * Dk * 32 + kBwStep * 32; }

// Chunked tensor-core backward (bf16, Dk = Dv = 128): what the reverse chain
// and the gradient assembly need after the forward's two passes ran with
// ForwardArgs::ckpt = ckpt.
struct BackwardTcArgs {
    const void *q, *k, *v, *log_alpha, *beta, *d_out;   // bf16
    const float *dS_final;            // or null
    const int32_t *cu_seqlens;
    float *dq, *dk, *dv, *dla, *dbeta;
    float *dS0;                       // or null
    int N, T, H;
    int32_t *status, *order, *chunk_off;
    const unsigned char *packets;
    size_t packet_slots;
    float *ckpt;                      // [slots, Dk, Dv] state entering every chunk
    float *dxs;                       // [slots, Dk, Dv] Gam_L dS' of every chunk
};
cudaError_t launch_backward_tc(const BackwardTcArgs &a, cudaStream_t s);

cudaError_t launch_varlen_index(const ForwardArgs &a, cudaStream_t s);
cudaError_t launch_backward(const BackwardArgs &a, cudaStream_t s);
cudaError_t launch_prefill_simt(const ForwardArgs &a, cudaStream_t s);
bool prefill_tc_supported(const ForwardArgs &a);
cudaError_t launch_prefill_tc(const ForwardArgs &a, cudaStream_t s);
cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t s);
cudaError_t launch_prefill_two_pass(const ForwardArgs &a, cudaStream_t s);

// Two-pass tensor-core prefill: bytes of one key-side operand packet and the
// number of packets a problem can need (one per 64-token chunk and head).
constexpr size_t kPacketBytes = 66048;
inline size_t packet_slots_bound(int64_t T, int64_t N, int64_t H) {
    return (size_t)((T + kChunk - 1) / kChunk + N) * (size_t)H;
}

// Driver API function `name` resolved through the runtime (the library does
// not link libcuda), or null when the driver lacks it.
void *driver_fn(const char *name);

// Makes the device that owns the caller's tensors current for one API call
// and, when that meant a switch, restores the context that was current on
// entry (a primary context, a driver-API context the caller pushed, or none)
// when it goes out of scope, on every return path.
class DeviceGuard {
  public:
    DeviceGuard() = default;
    DeviceGuard(const DeviceGuard &) = delete;
    DeviceGuard &operator=(const DeviceGuard &) = delete;
    ~DeviceGuard();
    // Switch to `dev` (no-op when it is current already).  False when the
    // switch failed; the caller's context is restored either way.
    bool use(int dev);

  private:
    bool switched_ = false;
    CUcontext saved_ = nullptr;
};

// TMA descriptor of a bf16 [T, H, D] tensor with a box of {box_x, 1, 64}
// (innermost first) and a 32/64/128-byte swizzle (0 = none).
bool make_tmap_bf16_3d(CUtensorMap *m, const void *base, int T, int H, int D, int box_x,
                       int swizzle_bytes);

// ---------------------------------------------------------------------------
// small device helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// In-chunk cumulative decay exp(-80): the smallest Gam the chunked
// factorisation exp(g_r - g_s) = Gam_r / Gam_s keeps inside fp32 range.
constexpr float kMinChunkDecay = 1.8048513e-35f;

// Record the first error code seen by any thread; later codes are dropped.
__device__ __forceinline__ void set_status(int32_t *status, int32_t code) {
    if (status) atomicCAS(status, 0, code);
}

// Index checks of the bounds-checking build (-DKDA_DEBUG_BOUNDS): a global
// access whose index would leave its buffer is skipped and KDA_ERR_BOUNDS is
// recorded in the status word (no trap).  In the regular build the check is
// the constant true and compiles away.
__device__ __forceinline__ bool debug_in_range(bool ok, int32_t *status) {
    if (!ok) set_status(status, KDA_ERR_BOUNDS);
    return ok;
}
#ifdef KDA_DEBUG_BOUNDS
#define KDA_IN_RANGE(cond, status) ::kda::debug_in_range((cond), (status))
#else
#define KDA_IN_RANGE(cond, status) true
#endif

// Token range of sequence n, or false when cu_seqlens is malformed there.
__device__ __forceinline__ bool seq_range(const int32_t *cu, int n, int T, int &t0, int &t1) {
    t0 = cu[n];
    t1 = cu[n + 1];
    return t0 >= 0 && t1 >= t0 && t1 <= T;
}

}  // namespace kda
