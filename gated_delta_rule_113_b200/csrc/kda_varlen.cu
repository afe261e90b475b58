// kda_varlen.cu -- varlen index: validate cu_seqlens and order the sequences.
//
// Packed sequences are delimited by cu_seqlens (sequence n owns tokens
// cu[n] .. cu[n+1]-1).  One block checks that the offsets start at 0, never
// decrease and end at total_tokens, records KDA_ERR_SEQLENS in the workspace
// status word otherwise, and writes a work order with the longest sequences
// first so the chain kernels start the longest sequential chains earliest.
// Running on the device keeps the whole call free of host synchronisation.
#include "kda_internal.cuh"

namespace kda {

__global__ void __launch_bounds__(1024) varlen_index_kernel(const int32_t *__restrict__ cu, int N,
                                                            int T, int32_t *status,
                                                            int32_t *order) {
    __shared__ int32_t s_len[kSortMax];
    __shared__ int s_bad;
    const int tid = threadIdx.x;
    if (tid == 0) {
        s_bad = (cu[0] != 0 || cu[N] != T) ? 1 : 0;
    }
    __syncthreads();
    for (int i = tid; i < N; i += blockDim.x) {
        const int a = cu[i], b = cu[i + 1];
        const bool ok = a >= 0 && b >= a && b <= T;
        if (!ok) s_bad = 1;
        if (N <= kSortMax) s_len[i] = ok ? (b - a) : 0;
    }
    __syncthreads();
    if (tid == 0) *status = s_bad ? KDA_ERR_SEQLENS : KDA_OK;
    if (N > kSortMax) {
        for (int i = tid; i < N; i += blockDim.x) order[i] = i;
        return;
    }
    // Rank sort: position of i = number of sequences strictly before it in
    // (length descending, index ascending) order.  A permutation by design.
    for (int i = tid; i < N; i += blockDim.x) {
        const int li = s_len[i];
        int rank = 0;
        for (int j = 0; j < N; ++j) {
            const int lj = s_len[j];
            rank += (lj > li) || (lj == li && j < i);
        }
        order[rank] = i;
    }
}

cudaError_t launch_varlen_index(const ForwardArgs &a, cudaStream_t s) {
    varlen_index_kernel<<<1, 1024, 0, s>>>(a.cu_seqlens, a.N, a.T, a.status, a.order);
    return cudaGetLastError();
}

}  // namespace kda
