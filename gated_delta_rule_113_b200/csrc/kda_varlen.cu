// kda_varlen.cu -- varlen index: validate cu_seqlens and order the sequences.
//
// Packed sequences are delimited by cu_seqlens (sequence n owns tokens
// cu[n] .. cu[n+1]-1).  One block checks that the offsets start at 0, never
// decrease and end at total_tokens, records KDA_ERR_SEQLENS in the workspace
// status word otherwise, and writes a work order with the longest sequences
// first so the chain kernels start the longest sequential chains earliest.
// Running on the device keeps the whole call free of host synchronisation.
#include "kda_internal.cuh"
#include "sm100.cuh"

namespace kda {

__global__ void __launch_bounds__(1024) varlen_index_kernel(const int32_t *__restrict__ cu, int N,
                                                            int T, int32_t *status,
                                                            int32_t *order, int32_t *chunk_off,
                                                            int32_t *work_ctr) {
    __shared__ int32_t s_len[kSortMax];
    __shared__ long long s_part[1024];
    __shared__ int s_bad;
    __shared__ int s_sat;
    const int tid = threadIdx.x;
    sm100::grid_launch_dependents();   // the key-side pass may start its set-up now
    if (tid == 0) s_sat = 0;
    if (chunk_off) {
        // chunk_off[n] = sum_{i<n} ceil(len_i / 64) (malformed sequences count
        // as empty): each thread scans a contiguous segment, then the block
        // scans the segment totals.  Well-formed offsets keep the sums below
        // T / 64 + N; overlapping (malformed) ones can push them past int32,
        // so they are formed in 64 bits and stored saturated at INT32_MAX,
        // which every consumer rejects as out of range.
        const int seg = (N + blockDim.x - 1) / blockDim.x;
        const int lo = tid * seg, hi = min(N, lo + seg);
        long long sum = 0;
        for (int i = lo; i < hi; ++i) {
            const int a = cu[i], b = cu[i + 1];
            if (a >= 0 && b >= a && b <= T) sum += (b - a + kChunk - 1) / kChunk;
        }
        s_part[tid] = sum;
        __syncthreads();
        // exclusive scan of the segment totals (Hillis-Steele, log2(1024) steps)
        for (int off = 1; off < (int)blockDim.x; off <<= 1) {
            const long long x = tid >= off ? s_part[tid - off] : 0;
            __syncthreads();
            s_part[tid] += x;
            __syncthreads();
        }
        const long long incl = s_part[tid];
        __syncthreads();
        s_part[tid] = incl - sum;
        __syncthreads();
        long long run = s_part[tid];
        bool sat = false;
        auto store = [&](int i, long long x) {
            if (x > 0x7fffffffLL) {
                x = 0x7fffffffLL;
                sat = true;
            }
            chunk_off[i] = (int32_t)x;
        };
        for (int i = lo; i < hi; ++i) {
            store(i, run);
            const int a = cu[i], b = cu[i + 1];
            if (a >= 0 && b >= a && b <= T) run += (b - a + kChunk - 1) / kChunk;
        }
        if (hi == N && lo < hi) store(N, run);
        if (N == 0 && tid == 0) chunk_off[0] = 0;
        if (sat) s_sat = 1;
        __syncthreads();
    }
    if (tid == 0) {
        s_bad = (cu[0] != 0 || cu[N] != T || s_sat) ? 1 : 0;
        if (work_ctr) *work_ctr = 0;   // the key-side pass claims items from here
    }
    __syncthreads();
    for (int i = tid; i < N; i += blockDim.x) {
        const int a = cu[i], b = cu[i + 1];
        const bool ok = a >= 0 && b >= a && b <= T;
        if (!ok) s_bad = 1;
        if (N <= kSortMax) s_len[i] = ok ? (b - a) : 0;
    }
    __syncthreads();
    if (tid == 0) {
        *status = s_bad ? KDA_ERR_SEQLENS : KDA_OK;
        status[8] = 0;   // where a bounded wait gave up, if one does (see report_abort)
        status[9] = 0;
    }
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
        if (KDA_IN_RANGE(rank < N, status)) order[rank] = i;
    }
}

cudaError_t launch_varlen_index(const ForwardArgs &a, cudaStream_t s) {
    varlen_index_kernel<<<1, 1024, 0, s>>>(a.cu_seqlens, a.N, a.T, a.status, a.order,
                                           a.chunk_off, a.work_ctr);
    return cudaGetLastError();
}

}  // namespace kda
