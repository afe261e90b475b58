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
//     address is looked up once per device with cudaGetSymbolAddress, with
//     that device current, on the first call that uses the device; that first
//     call should therefore come before any stream capture.
//   - All calls share the one array.  Each call rewrites what it needs before
//     use (the status word is reset by the first kernel of the call), but
//     calls whose kernels overlap on the GPU race on it: order them on one
//     stream, or serialise them otherwise.
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
void *g_scratch_addr[kMaxDevices];   // device address of the array, per device
std::mutex g_scratch_mu;

// Make the device that owns `probe` current and return the array's device
// address on it, looking it up on first use.
kda_status scratch_on_device_of(const void *probe, void **addr) {
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, probe) != cudaSuccess) {
        cudaGetLastError();
        return KDA_ERR_INVALID;
    }
    if (at.type != cudaMemoryTypeDevice && at.type != cudaMemoryTypeManaged)
        return KDA_ERR_INVALID;
    const int dev = at.device;
    if (dev < 0 || dev >= kMaxDevices) return KDA_ERR_UNSUPPORTED;
    int cur = -1;
    if (cudaGetDevice(&cur) != cudaSuccess) return KDA_ERR_CUDA;
    if (cur != dev && cudaSetDevice(dev) != cudaSuccess) return KDA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            return KDA_ERR_CUDA;
        }
        g_scratch_addr[dev] = p;
    }
    *addr = g_scratch_addr[dev];
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
    void *scratch = nullptr;
    const kda_status st = scratch_on_device_of(probe, &scratch);
    if (st != KDA_OK) return st;
    return kda_forward(q, k, v, log_alpha, beta, S0, cu_seqlens, out, S_final, p, scratch,
                       kScratchBytes, stream);
}
