// kda_noalloc.cu -- kda_forward for callers that cannot allocate device memory.
//
// kda_forward needs a small device workspace (a status word and the
// per-sequence work order).  Some callers have no way to provide one: an
// engine whose device memory is fully planned ahead of time and that forbids
// allocation on its serving path, a plug-in running inside a host
// application that owns the allocator, or a latency-critical path that must
// not take cudaMalloc's implicit device synchronisation.  This entry point
// serves them from a fixed scratch array that lives in the library itself:
//
//   - The array is a file-scope __device__ variable, so every GPU that loads
//     the library holds its bytes (KDA_NOALLOC_MAX_SEQS int32 entries plus a
//     256-byte header) until the process exits.
//   - In host code the array's name is only a host-side stand-in.  Its device
//     address is looked up with cudaGetSymbolAddress, with the device current,
//     on the first call that uses a device, and cached per device together
//     with the identity of the CUDA context it was looked up in; a call made
//     under another context of that device (a driver-API context the caller
//     pushed, or the primary context re-created after cudaDeviceReset) looks
//     it up again.  The first call on a device (and in a context) should
//     therefore come before any stream capture.
//   - All calls share the one array.  Each call rewrites what it needs before
//     use (the status word is reset by the first kernel of the call), but
//     calls whose kernels overlap on the GPU race on it: order them on one
//     stream, or serialise them otherwise.  kda_forward_noalloc_status reads
//     the status word the last call on a device left there.
//   - Nothing here calls cudaMalloc, cudaFree or any allocating routine; the
//     kernels and checks are exactly those of kda_forward, which this entry
//     point calls with the scratch array as its workspace.
#include <mutex>

#include "kda_internal.cuh"

namespace {

constexpr size_t kScratchBytes =
    kda::kWsHeader + sizeof(int32_t) * (size_t)KDA_NOALLOC_MAX_SEQS;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
struct ScratchAddr {
    unsigned long long ctx_id;   // context the address was looked up in (0: none yet)
    void *addr;
};
ScratchAddr g_scratch[kMaxDevices];
std::mutex g_scratch_mu;

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

// Identity of the calling thread's current context: its unique id where the
// driver has cuCtxGetId, else its handle.  0 when none can be had.
unsigned long long current_ctx_id() {
    static CtxGetCurrentFn get_cur = reinterpret_cast<CtxGetCurrentFn>(kda::driver_fn("cuCtxGetCurrent"));
    static CtxGetIdFn get_id = reinterpret_cast<CtxGetIdFn>(kda::driver_fn("cuCtxGetId"));
    CUcontext ctx = nullptr;
    if (!get_cur || get_cur(&ctx) != CUDA_SUCCESS || !ctx) return 0;
    unsigned long long id = 0;
    if (get_id && get_id(ctx, &id) == CUDA_SUCCESS && id) return id;
    return (unsigned long long)(uintptr_t)ctx;
}

// Make the device that owns `probe` current (through `guard`, which puts the
// caller's context back later) and return the array's device address in the
// context now current, looking it up when this device and context have not
// been seen before.
kda_status scratch_on_device_of(const void *probe, kda::DeviceGuard &guard, void **addr) {
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, probe) != cudaSuccess) {
        cudaGetLastError();
        return KDA_ERR_INVALID;
    }
    if (at.type != cudaMemoryTypeDevice && at.type != cudaMemoryTypeManaged)
        return KDA_ERR_INVALID;
    const int dev = at.device;
    if (dev < 0 || dev >= kMaxDevices) return KDA_ERR_UNSUPPORTED;
    if (!guard.use(dev)) return KDA_ERR_CUDA;
    const unsigned long long ctx = current_ctx_id();
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    ScratchAddr &e = g_scratch[dev];
    if (!e.addr || ctx == 0 || e.ctx_id != ctx) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            e.addr = nullptr;
            return KDA_ERR_CUDA;
        }
        e.addr = p;
        e.ctx_id = ctx;
    }
    *addr = e.addr;
    return KDA_OK;
}

}  // namespace

extern "C" kda_status kda_forward_noalloc(const void *q, const void *k, const void *v,
                                          const void *log_alpha, const void *beta,
                                          const float *S0, const int32_t *cu_seqlens,
                                          void *out, float *S_final, const kda_params *p,
                                          void *stream) {
    if (!p) return KDA_ERR_INVALID;
    if (p->num_seqs > KDA_NOALLOC_MAX_SEQS) return KDA_ERR_UNSUPPORTED;
    if (p->num_seqs <= 0)  // nothing to run: same answer as kda_forward
        return kda_forward(q, k, v, log_alpha, beta, S0, cu_seqlens, out, S_final, p, nullptr,
                           0, stream);
    const void *probe = cu_seqlens ? (const void *)cu_seqlens : out;
    if (!probe) return KDA_ERR_INVALID;
    kda::DeviceGuard guard;
    void *scratch = nullptr;
    const kda_status st = scratch_on_device_of(probe, guard, &scratch);
    if (st != KDA_OK) return st;
    return kda_forward(q, k, v, log_alpha, beta, S0, cu_seqlens, out, S_final, p, scratch,
                       kScratchBytes, stream);
}

extern "C" kda_status kda_forward_noalloc_status(const void *device_ptr, int32_t *status,
                                                 void *stream) {
    if (!device_ptr || !status) return KDA_ERR_INVALID;
    kda::DeviceGuard guard;
    void *scratch = nullptr;
    const kda_status st = scratch_on_device_of(device_ptr, guard, &scratch);
    if (st != KDA_OK) return st;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess ||
        cudaMemcpy(status, scratch, sizeof(int32_t), cudaMemcpyDeviceToHost) != cudaSuccess) {
        cudaGetLastError();
        return KDA_ERR_CUDA;
    }
    return KDA_OK;
}
