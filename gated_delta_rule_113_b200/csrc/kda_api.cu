// kda_api.cu -- the C ABI declared in include/kda.h: host validation,
// workspace layout, device selection and kernel dispatch.
#include <string.h>

#include "kda_internal.cuh"

namespace {

using kda::kWsHeader;

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }
size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool dtype_ok(int32_t d) { return d == KDA_F32 || d == KDA_BF16; }
bool width_ok(int32_t d) { return d == 64 || d == 128; }

kda_status check_common(const kda_params *p) {
    if (!p) return KDA_ERR_INVALID;
    if (p->num_seqs < 0 || p->H <= 0) return KDA_ERR_INVALID;
    if (!dtype_ok(p->io_dtype) || !dtype_ok(p->gate_dtype)) return KDA_ERR_UNSUPPORTED;
    if (!width_ok(p->Dk) || !width_ok(p->Dv)) return KDA_ERR_UNSUPPORTED;
    if (p->flags & ~(KDA_FLAG_FORCE_SIMT | KDA_FLAG_FUSED_TC | KDA_FLAG_TEST_STALL))
        return KDA_ERR_INVALID;
    return KDA_OK;
}

// Pointers must be device (or managed) memory of one device; make that
// device current for the launches (the guard restores the caller's context
// when the entry point returns).  Host memory would fault on the GPU.
kda_status select_device(const void *const *ptrs, int n, kda::DeviceGuard &guard) {
    int dev = -1;
    for (int i = 0; i < n; ++i) {
        if (!ptrs[i]) continue;
        cudaPointerAttributes at;
        if (cudaPointerGetAttributes(&at, ptrs[i]) != cudaSuccess) {
            cudaGetLastError();
            return KDA_ERR_INVALID;
        }
        if (at.type != cudaMemoryTypeDevice && at.type != cudaMemoryTypeManaged)
            return KDA_ERR_INVALID;
        if (dev < 0) dev = at.device;
        else if (dev != at.device) return KDA_ERR_INVALID;
    }
    if (dev < 0) return KDA_OK;
    return guard.use(dev) ? KDA_OK : KDA_ERR_CUDA;
}

// Workspace layout: [status header][order: N int32][chunk_off: N+1 int32]
// [operand packets].  The first two parts are always needed; the last two
// only by the two-pass tensor-core prefill.
size_t workspace_bytes(const kda_params *p) {
    return kWsHeader + round_up(sizeof(int32_t) * (size_t)p->num_seqs, 256);
}

bool tc_shape(const kda_params *p) {
    return p->io_dtype == KDA_BF16 && p->gate_dtype == KDA_BF16 && p->Dk == 128 && p->Dv == 128;
}

size_t chunk_off_offset(const kda_params *p) { return workspace_bytes(p); }

size_t packets_offset(const kda_params *p) {
    return chunk_off_offset(p) + round_up(sizeof(int32_t) * ((size_t)p->num_seqs + 1), 256);
}

size_t workspace_bytes_two_pass(const kda_params *p) {
    return packets_offset(p) +
           kda::packet_slots_bound(p->total_tokens, p->num_seqs, p->H) * kda::kPacketBytes;
}

}  // namespace

extern "C" {

int32_t kda_abi_version(void) { return KDA_ABI_VERSION; }

const char *kda_status_string(kda_status s) {
    switch (s) {
    case KDA_OK: return "KDA_OK";
    case KDA_ERR_INVALID: return "KDA_ERR_INVALID: invalid argument";
    case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED: unsupported shape or dtype";
    case KDA_ERR_ALIGN: return "KDA_ERR_ALIGN: tensor not 16-byte aligned";
    case KDA_ERR_WORKSPACE: return "KDA_ERR_WORKSPACE: workspace missing, misaligned or too small";
    case KDA_ERR_CUDA: return "KDA_ERR_CUDA: CUDA call or launch failed";
    case KDA_ERR_TIMEOUT: return "KDA_ERR_TIMEOUT: bounded device wait gave up";
    case KDA_ERR_SEQLENS: return "KDA_ERR_SEQLENS: cu_seqlens not monotone from 0 to total_tokens";
    case KDA_ERR_SLOT: return "KDA_ERR_SLOT: snapshot-pool slot outside the pool";
    case KDA_ERR_DECAY:
        return "KDA_ERR_DECAY: log_alpha > 0 or not finite, or in-chunk cumulative log-decay below -80";
    case KDA_ERR_BOUNDS: return "KDA_ERR_BOUNDS: index outside its buffer (bounds-checking build)";
    }
    return "KDA_ERR_UNKNOWN";
}

size_t kda_forward_workspace_size(const kda_params *p) {
    if (check_common(p) != KDA_OK) return 0;
    if (tc_shape(p) && !(p->flags & (KDA_FLAG_FORCE_SIMT | KDA_FLAG_FUSED_TC)) &&
        p->total_tokens >= 0)
        return workspace_bytes_two_pass(p);
    return workspace_bytes(p);
}

namespace {

kda_status forward_impl(const void *q, const void *k, const void *v, const void *log_alpha,
                        const void *beta, const float *S0, const int32_t *cu_seqlens, void *out,
                        float *S_final, const kda_params *p, const kda_snapshots *snap,
                        void *workspace, size_t ws_bytes, void *stream) {
    kda_status st = check_common(p);
    if (st != KDA_OK) return st;
    if (p->chunk != kda::kChunk || p->total_tokens < 0) return KDA_ERR_UNSUPPORTED;
    if (p->num_seqs == 0) return p->total_tokens == 0 ? KDA_OK : KDA_ERR_INVALID;
    if (!cu_seqlens) return KDA_ERR_INVALID;
    if (p->total_tokens > 0 && (!q || !k || !v || !log_alpha || !beta || !out))
        return KDA_ERR_INVALID;
    // snapshots: `every` a multiple of the chunk; pool and slot arrays present
    const bool use_snap = snap && (snap->every != 0 || snap->s0_slot);
    if (use_snap) {
        if (snap->every < 0 || snap->every % kda::kChunk) return KDA_ERR_INVALID;
        if (!snap->pool || snap->n_slots <= 0) return KDA_ERR_INVALID;
        if (snap->every > 0 && !snap->slot_base) return KDA_ERR_INVALID;
        if (!aligned16(snap->pool)) return KDA_ERR_ALIGN;
    }
    const void *ptrs[] = {q, k, v, log_alpha, beta, S0, cu_seqlens, out, S_final, workspace,
                          use_snap ? snap->pool : nullptr,
                          use_snap ? snap->slot_base : nullptr,
                          use_snap ? snap->s0_slot : nullptr};
    for (int i = 0; i < 10; ++i)
        if (ptrs[i] && !aligned16(ptrs[i])) return KDA_ERR_ALIGN;
    if (!workspace || ((uintptr_t)workspace & 255u) || ws_bytes < workspace_bytes(p))
        return KDA_ERR_WORKSPACE;
    // grid = N * H * (Dv / 32) CTAs must fit in gridDim.x
    if ((long long)p->num_seqs * p->H * (p->Dv / 32) > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;
    kda::DeviceGuard guard;
    st = select_device(ptrs, 13, guard);
    if (st != KDA_OK) return st;

    kda::ForwardArgs a;
    a.q = q; a.k = k; a.v = v; a.log_alpha = log_alpha; a.beta = beta;
    a.S0 = S0; a.cu_seqlens = cu_seqlens; a.out = out; a.S_final = S_final;
    a.N = p->num_seqs; a.T = p->total_tokens; a.H = p->H; a.Dk = p->Dk; a.Dv = p->Dv;
    a.io_dtype = p->io_dtype; a.gate_dtype = p->gate_dtype;
    a.status = reinterpret_cast<int32_t *>(workspace);
    a.work_ctr = a.status + 4;   // inside the 256-byte header
    a.order = reinterpret_cast<int32_t *>(static_cast<char *>(workspace) + kWsHeader);
    a.chunk_off = nullptr;
    a.packets = nullptr;
    a.packet_slots = 0;
    a.snap_pool = use_snap ? snap->pool : nullptr;
    a.snap_base = use_snap && snap->every > 0 ? snap->slot_base : nullptr;
    a.s0_slot = use_snap ? snap->s0_slot : nullptr;
    a.snap_slots = use_snap ? (long long)snap->n_slots : 0;
    a.snap_every_chunks = use_snap ? snap->every / kda::kChunk : 0;
    a.test_stall = (p->flags & KDA_FLAG_TEST_STALL) != 0;
    a.ckpt = nullptr;

    // bf16 with Dk = Dv = 128: tensor cores, two-pass when the workspace holds
    // the operand packets, else the single fused kernel; otherwise CUDA cores.
    const bool tc = !(p->flags & KDA_FLAG_FORCE_SIMT) && kda::prefill_tc_supported(a);
    const bool two_pass =
        tc && !(p->flags & KDA_FLAG_FUSED_TC) && ws_bytes >= workspace_bytes_two_pass(p);
    if (use_snap && !two_pass) return KDA_ERR_UNSUPPORTED;   // only the chain pass keeps them
    if (two_pass) {
        char *ws = static_cast<char *>(workspace);
        a.chunk_off = reinterpret_cast<int32_t *>(ws + chunk_off_offset(p));
        a.packets = reinterpret_cast<unsigned char *>(ws + packets_offset(p));
        a.packet_slots = kda::packet_slots_bound(p->total_tokens, p->num_seqs, p->H);
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (kda::launch_varlen_index(a, s) != cudaSuccess) return KDA_ERR_CUDA;
    cudaError_t e;
    if (two_pass) e = kda::launch_prefill_two_pass(a, s);
    else if (tc) e = kda::launch_prefill_tc(a, s);
    else e = kda::launch_prefill_simt(a, s);
    if (e != cudaSuccess) return KDA_ERR_CUDA;
    return KDA_OK;
}

}  // namespace

kda_status kda_forward(const void *q, const void *k, const void *v, const void *log_alpha,
                       const void *beta, const float *S0, const int32_t *cu_seqlens, void *out,
                       float *S_final, const kda_params *p, void *workspace, size_t ws_bytes,
                       void *stream) {
    return forward_impl(q, k, v, log_alpha, beta, S0, cu_seqlens, out, S_final, p, nullptr,
                        workspace, ws_bytes, stream);
}

kda_status kda_forward_snapshots(const void *q, const void *k, const void *v,
                                 const void *log_alpha, const void *beta, const float *S0,
                                 const int32_t *cu_seqlens, void *out, float *S_final,
                                 const kda_params *p, const kda_snapshots *snap, void *workspace,
                                 size_t ws_bytes, void *stream) {
    return forward_impl(q, k, v, log_alpha, beta, S0, cu_seqlens, out, S_final, p, snap,
                        workspace, ws_bytes, stream);
}

kda_status kda_decode_step(const void *q, const void *k, const void *v, const void *log_alpha,
                           const void *beta, float *S, void *out, const kda_params *p,
                           void *stream) {
    kda_status st = check_common(p);
    if (st != KDA_OK) return st;
    if (p->num_seqs == 0) return KDA_OK;
    if (!q || !k || !v || !log_alpha || !beta || !S || !out) return KDA_ERR_INVALID;
    const void *ptrs[] = {q, k, v, log_alpha, beta, S, out};
    for (const void *x : ptrs)
        if (!aligned16(x)) return KDA_ERR_ALIGN;
    if ((long long)p->num_seqs * p->H * (p->Dv / 64) > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;
    kda::DeviceGuard guard;
    st = select_device(ptrs, 7, guard);
    if (st != KDA_OK) return st;

    kda::DecodeArgs a;
    a.q = q; a.k = k; a.v = v; a.log_alpha = log_alpha; a.beta = beta; a.S = S; a.out = out;
    a.S_tokens = nullptr;
    a.n_tokens = 1;
    a.N = p->num_seqs; a.H = p->H; a.Dk = p->Dk; a.Dv = p->Dv;
    a.io_dtype = p->io_dtype; a.gate_dtype = p->gate_dtype;
    if (kda::launch_decode(a, static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return KDA_ERR_CUDA;
    return KDA_OK;
}

kda_status kda_decode_multi(const void *q, const void *k, const void *v, const void *log_alpha,
                            const void *beta, const float *S, float *S_tokens, void *out,
                            const kda_params *p, int32_t n_tokens, void *stream) {
    kda_status st = check_common(p);
    if (st != KDA_OK) return st;
    if (n_tokens < 1) return KDA_ERR_INVALID;
    if (p->num_seqs == 0) return KDA_OK;
    if (!q || !k || !v || !log_alpha || !beta || !S || !S_tokens || !out) return KDA_ERR_INVALID;
    const void *ptrs[] = {q, k, v, log_alpha, beta, S, S_tokens, out};
    for (const void *x : ptrs)
        if (!aligned16(x)) return KDA_ERR_ALIGN;
    if ((long long)p->num_seqs * p->H * (p->Dv / 64) > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;
    if ((long long)p->num_seqs * n_tokens > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;
    kda::DeviceGuard guard;
    st = select_device(ptrs, 8, guard);
    if (st != KDA_OK) return st;

    kda::DecodeArgs a;
    a.q = q; a.k = k; a.v = v; a.log_alpha = log_alpha; a.beta = beta;
    a.S = const_cast<float *>(S);   // only read when S_tokens is set
    a.S_tokens = S_tokens;
    a.n_tokens = n_tokens;
    a.out = out;
    a.N = p->num_seqs; a.H = p->H; a.Dk = p->Dk; a.Dv = p->Dv;
    a.io_dtype = p->io_dtype; a.gate_dtype = p->gate_dtype;
    if (kda::launch_decode(a, static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return KDA_ERR_CUDA;
    return KDA_OK;
}

// Backward workspace: [status header][order: N int32][chunk_off: N+1 int32]
// [states every 32 tokens: 2 (ceil(T/64) + N) x H x Dk x Dv fp32]
// [per-CTA scratch: N x H x Dv/32 CTAs]
// [per value slice: partial dq, dk, dlog_alpha, dbeta].
namespace {
size_t bw_ckpt_steps(const kda_params *p) {
    return 2 * ((size_t)((p->total_tokens + kda::kChunk - 1) / kda::kChunk) + (size_t)p->num_seqs);
}
size_t bw_ckpt_offset(const kda_params *p) {
    return kWsHeader + round_up(sizeof(int32_t) * (size_t)p->num_seqs, 256) +
           round_up(sizeof(int32_t) * ((size_t)p->num_seqs + 1), 256);
}
size_t bw_scratch_offset(const kda_params *p) {
    return bw_ckpt_offset(p) +
           round_up(bw_ckpt_steps(p) * p->H * p->Dk * p->Dv * sizeof(float), 256);
}
size_t bw_part_offset(const kda_params *p) {
    const size_t ctas = (size_t)p->num_seqs * p->H * (p->Dv / 32);
    return bw_scratch_offset(p) +
           round_up(ctas * kda::backward_scratch_floats(p->Dk) * sizeof(float), 256);
}
size_t bw_workspace_bytes(const kda_params *p) {
    return bw_part_offset(p) + (size_t)(p->Dv / 32) *
                                   kda::backward_part_floats(p->total_tokens, p->H, p->Dk) *
                                   sizeof(float);
}

// Chunked tensor-core backward workspace: [header][order][chunk_off][packets]
// [state entering every chunk][Gam_L dS' of every chunk], one 64 KB fp32
// state per (chunk, head) in each of the last two.
size_t bw_tc_ckpt_offset(const kda_params *p) {
    return packets_offset(p) +
           kda::packet_slots_bound(p->total_tokens, p->num_seqs, p->H) * kda::kPacketBytes;
}
size_t bw_tc_state_bytes(const kda_params *p) {
    return kda::packet_slots_bound(p->total_tokens, p->num_seqs, p->H) * (size_t)p->Dk * p->Dv *
           sizeof(float);
}
size_t bw_tc_workspace_bytes(const kda_params *p) {
    return bw_tc_ckpt_offset(p) + 2 * bw_tc_state_bytes(p);
}
bool bw_tc_path(const kda_params *p) { return tc_shape(p) && !(p->flags & KDA_FLAG_FORCE_SIMT); }
}  // namespace

size_t kda_backward_workspace_size(const kda_params *p) {
    if (check_common(p) != KDA_OK || p->total_tokens < 0) return 0;
    return bw_tc_path(p) ? bw_tc_workspace_bytes(p) : bw_workspace_bytes(p);
}

namespace {
// The chunked tensor-core backward: the varlen index, the forward's two
// passes keeping every chunk's entering state (no output), then the reverse
// chain and the gradient assembly.
kda_status backward_tc(const void *q, const void *k, const void *v, const void *log_alpha,
                       const void *beta, const float *S0, const int32_t *cu_seqlens,
                       const void *d_out, const float *dS_final, float *dq, float *dk, float *dv,
                       float *dlog_alpha, float *dbeta, float *dS0, const kda_params *p,
                       void *workspace, cudaStream_t s) {
    char *ws = static_cast<char *>(workspace);
    kda::ForwardArgs a;
    memset(&a, 0, sizeof(a));
    a.q = q; a.k = k; a.v = v; a.log_alpha = log_alpha; a.beta = beta;
    a.S0 = S0; a.cu_seqlens = cu_seqlens; a.out = nullptr; a.S_final = nullptr;
    a.N = p->num_seqs; a.T = p->total_tokens; a.H = p->H; a.Dk = p->Dk; a.Dv = p->Dv;
    a.io_dtype = p->io_dtype; a.gate_dtype = p->gate_dtype;
    a.status = reinterpret_cast<int32_t *>(ws);
    a.work_ctr = a.status + 4;
    a.order = reinterpret_cast<int32_t *>(ws + kWsHeader);
    a.chunk_off = reinterpret_cast<int32_t *>(ws + chunk_off_offset(p));
    a.packets = reinterpret_cast<unsigned char *>(ws + packets_offset(p));
    a.packet_slots = kda::packet_slots_bound(p->total_tokens, p->num_seqs, p->H);
    a.ckpt = reinterpret_cast<float *>(ws + bw_tc_ckpt_offset(p));
    if (kda::launch_varlen_index(a, s) != cudaSuccess) return KDA_ERR_CUDA;
    if (p->total_tokens > 0 && kda::launch_prefill_two_pass(a, s) != cudaSuccess) return KDA_ERR_CUDA;
    kda::BackwardTcArgs b;
    b.q = q; b.k = k; b.v = v; b.log_alpha = log_alpha; b.beta = beta; b.d_out = d_out;
    b.dS_final = dS_final; b.cu_seqlens = cu_seqlens;
    b.dq = dq; b.dk = dk; b.dv = dv; b.dla = dlog_alpha; b.dbeta = dbeta; b.dS0 = dS0;
    b.N = p->num_seqs; b.T = p->total_tokens; b.H = p->H;
    b.status = a.status; b.order = a.order; b.chunk_off = a.chunk_off;
    b.packets = a.packets; b.packet_slots = a.packet_slots;
    b.ckpt = a.ckpt;
    b.dxs = reinterpret_cast<float *>(ws + bw_tc_ckpt_offset(p) + bw_tc_state_bytes(p));
    if (p->total_tokens > 0) {
        if (kda::launch_backward_tc(b, s) != cudaSuccess) return KDA_ERR_CUDA;
    } else if (dS0) {
        // no tokens: dS0 = dS_final (or zero), sequence by sequence
        const size_t bytes = (size_t)p->num_seqs * p->H * p->Dk * p->Dv * sizeof(float);
        const cudaError_t e = dS_final ? cudaMemcpyAsync(dS0, dS_final, bytes, cudaMemcpyDeviceToDevice, s)
                                       : cudaMemsetAsync(dS0, 0, bytes, s);
        if (e != cudaSuccess) return KDA_ERR_CUDA;
    }
    return KDA_OK;
}
}  // namespace

kda_status kda_backward(const void *q, const void *k, const void *v, const void *log_alpha,
                        const void *beta, const float *S0, const int32_t *cu_seqlens,
                        const void *d_out, const float *dS_final, float *dq, float *dk,
                        float *dv, float *dlog_alpha, float *dbeta, float *dS0,
                        const kda_params *p, void *workspace, size_t ws_bytes, void *stream) {
    kda_status st = check_common(p);
    if (st != KDA_OK) return st;
    if (p->chunk != kda::kChunk || p->total_tokens < 0) return KDA_ERR_UNSUPPORTED;
    if (p->num_seqs == 0) return p->total_tokens == 0 ? KDA_OK : KDA_ERR_INVALID;
    if (!cu_seqlens) return KDA_ERR_INVALID;
    if (p->total_tokens > 0 && (!q || !k || !v || !log_alpha || !beta || !d_out || !dq || !dk ||
                                !dv || !dlog_alpha || !dbeta))
        return KDA_ERR_INVALID;
    const void *ptrs[] = {q, k, v, log_alpha, beta, S0, cu_seqlens, d_out, dS_final, dq, dk,
                          dv, dlog_alpha, dbeta, dS0, workspace};
    for (const void *x : ptrs)
        if (x && !aligned16(x)) return KDA_ERR_ALIGN;
    const bool tc_path = bw_tc_path(p);
    if (!workspace || ((uintptr_t)workspace & 255u) ||
        ws_bytes < (tc_path ? bw_tc_workspace_bytes(p) : bw_workspace_bytes(p)))
        return KDA_ERR_WORKSPACE;
    if ((long long)p->num_seqs * p->H * (p->Dv / 32) > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;
    kda::DeviceGuard guard;
    st = select_device(ptrs, 16, guard);
    if (st != KDA_OK) return st;
    if (tc_path)
        return backward_tc(q, k, v, log_alpha, beta, S0, cu_seqlens, d_out, dS_final, dq, dk, dv,
                           dlog_alpha, dbeta, dS0, p, workspace, static_cast<cudaStream_t>(stream));

    char *ws = static_cast<char *>(workspace);
    kda::ForwardArgs ix;   // the varlen index: validation, order, chunk offsets
    memset(&ix, 0, sizeof(ix));
    ix.cu_seqlens = cu_seqlens;
    ix.N = p->num_seqs; ix.T = p->total_tokens; ix.H = p->H;
    ix.status = reinterpret_cast<int32_t *>(ws);
    ix.order = reinterpret_cast<int32_t *>(ws + kWsHeader);
    ix.chunk_off = reinterpret_cast<int32_t *>(
        ws + kWsHeader + round_up(sizeof(int32_t) * (size_t)p->num_seqs, 256));
    ix.work_ctr = nullptr;
    kda::BackwardArgs a;
    a.q = q; a.k = k; a.v = v; a.log_alpha = log_alpha; a.beta = beta; a.d_out = d_out;
    a.S0 = S0; a.dS_final = dS_final; a.cu_seqlens = cu_seqlens;
    a.dq = dq; a.dk = dk; a.dv = dv; a.dla = dlog_alpha; a.dbeta = dbeta; a.dS0 = dS0;
    a.N = p->num_seqs; a.T = p->total_tokens; a.H = p->H; a.Dk = p->Dk; a.Dv = p->Dv;
    a.io_dtype = p->io_dtype; a.gate_dtype = p->gate_dtype;
    a.status = ix.status; a.order = ix.order; a.chunk_off = ix.chunk_off;
    a.ckpt = reinterpret_cast<float *>(ws + bw_ckpt_offset(p));
    a.ckpt_steps = bw_ckpt_steps(p);
    a.scratch = reinterpret_cast<float *>(ws + bw_scratch_offset(p));
    a.part = reinterpret_cast<float *>(ws + bw_part_offset(p));
    a.part_stride = kda::backward_part_floats(p->total_tokens, p->H, p->Dk);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (kda::launch_varlen_index(ix, s) != cudaSuccess) return KDA_ERR_CUDA;
    if (kda::launch_backward(a, s) != cudaSuccess) return KDA_ERR_CUDA;
    return KDA_OK;
}

kda_status kda_workspace_status(const void *workspace, int32_t *status, void *stream) {
    if (!workspace || !status) return KDA_ERR_INVALID;
    const void *ptrs[] = {workspace};
    kda::DeviceGuard guard;
    kda_status st = select_device(ptrs, 1, guard);
    if (st != KDA_OK) return st;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return KDA_ERR_CUDA;
    if (cudaMemcpy(status, workspace, sizeof(int32_t), cudaMemcpyDeviceToHost) != cudaSuccess)
        return KDA_ERR_CUDA;
    return KDA_OK;
}

}  // extern "C"
