// umma_probe.cu -- test-only probe of the tcgen05.mma operand layouts the KDA
// prefill kernel relies on.  One CTA stages A (M x K) and B (K x N) in shared
// memory in a chosen major-ness / swizzle, issues K/16 MMAs into TMEM, and
// copies every TMEM lane x column back, so the host can compare D with A*B.
// With a_tmem, A is first written into tensor memory (columns 128 ..) by the
// four warps and the MMAs read it from there.
// Built and run only by tests/test_gpu_tcgen05_layouts.py.
#include <cuda_runtime.h>
#include <stdint.h>

#include "sm100.cuh"

using namespace kda::sm100;

struct ProbeCfg {
    int M, N, K;
    int a_mn;      // A stored MN-major (1) or K-major (0); always 128B swizzle
    int b_mn;      // B stored MN-major (1) or K-major (0)
    int b_swz;     // B swizzle: 128 or 64 (64 only for MN-major with N == 32)
    int neg_a;
    int a_tmem;    // A staged in tensor memory (packed bf16 pairs, lane = row) instead
};

// byte offset of A(m, k) and B(k, n) inside their tiles
__device__ uint32_t a_off(const ProbeCfg &c, int m, int k) {
    if (!c.a_mn) {  // K-major SW128: [k-atom][M rows][128 B]
        const uint32_t byte = (k % 64) * 2;
        return (k / 64) * (c.M * 128) + sw128_off(m, byte / 16) + byte % 16;
    }
    // MN-major SW128: [m-block of 64][K rows][128 B]
    const uint32_t byte = (m % 64) * 2;
    return (m / 64) * (c.K * 128) + sw128_off(k, byte / 16) + byte % 16;
}

__device__ uint32_t b_off(const ProbeCfg &c, int k, int n) {
    if (!c.b_mn) {  // K-major SW128: [k-atom][N rows][128 B]
        const uint32_t byte = (k % 64) * 2;
        return (k / 64) * (c.N * 128) + sw128_off(n, byte / 16) + byte % 16;
    }
    if (c.b_swz == 64) {  // MN-major SW64, N == 32: [K rows][64 B]
        const uint32_t byte = n * 2;
        return sw64_off(k, byte / 16) + byte % 16;
    }
    const uint32_t byte = (n % 64) * 2;  // MN-major SW128: [n-block][K rows][128 B]
    return (n / 64) * (c.K * 128) + sw128_off(k, byte / 16) + byte % 16;
}

__global__ void __launch_bounds__(128) probe_kernel(ProbeCfg c, const uint16_t *A,
                                                    const uint16_t *B, float *D, int *err) {
    extern __shared__ unsigned char smem_raw[];
    // swizzle atoms must sit on 1024-byte boundaries
    unsigned char *smem = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    unsigned char *sA = smem;                 // up to 32 KB
    unsigned char *sB = smem + 32768;         // up to 32 KB
    __shared__ uint64_t bar;
    __shared__ uint32_t tbase;
    const int tid = threadIdx.x, warp = tid / 32;

    for (int i = tid; i < c.M * c.K; i += 128) {
        const int m = i / c.K, k = i % c.K;
        *reinterpret_cast<uint16_t *>(sA + a_off(c, m, k)) = A[i];
    }
    for (int i = tid; i < c.K * c.N; i += 128) {
        const int k = i / c.N, n = i % c.N;
        *reinterpret_cast<uint16_t *>(sB + b_off(c, k, n)) = B[i];
    }
    fence_proxy_async();
    if (warp == 0) tmem_alloc(&tbase, 256);
    __syncthreads();
    if (c.a_tmem) {
        // lane m = tid holds row m of A: column 128 + j packs (A[m][2j], A[m][2j+1]),
        // the even element in the low half
        tc_fence_after();
        const int m = tid;
        for (int j0 = 0; j0 < c.K / 2; j0 += 16) {
            uint32_t r[16];
            for (int j = 0; j < 16; ++j) {
                const uint32_t lo = m < c.M ? A[m * c.K + 2 * (j0 + j)] : 0u;
                const uint32_t hi = m < c.M ? A[m * c.K + 2 * (j0 + j) + 1] : 0u;
                r[j] = lo | (hi << 16);
            }
            tmem_st16(tmem_addr(tbase, warp * 32, 128 + j0), r);
        }
        tmem_wait_st();
    }
    if (tid == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = tbase;

    if (tid == 0) {
        const uint32_t a0 = smem_u32(sA), b0 = smem_u32(sB);
        const uint32_t idesc = idesc_bf16(c.M, c.N, c.a_mn, c.b_mn, c.neg_a);
        for (int ks = 0; ks < c.K / 16; ++ks) {
            uint64_t ad = 0, bd;
            if (!c.a_mn) {
                ad = smem_desc(a0 + (ks / 4) * (c.M * 128) + (ks % 4) * 32, 16, 1024, kSw128);
            } else {
                ad = smem_desc(a0 + ks * 2048, c.K * 128, 1024, kSw128);
            }
            if (!c.b_mn) {
                bd = smem_desc(b0 + (ks / 4) * (c.N * 128) + (ks % 4) * 32, 16, 1024, kSw128);
            } else if (c.b_swz == 64) {
                bd = smem_desc(b0 + ks * 1024, c.K * 64, 512, kSw64);
            } else {
                bd = smem_desc(b0 + ks * 2048, c.K * 128, 1024, kSw128);
            }
            if (c.a_tmem) mma_bf16_ta(tm, tm + 128 + 8 * ks, bd, idesc, ks > 0 ? 1u : 0u);
            else mma_bf16(tm, ad, bd, idesc, ks > 0 ? 1u : 0u);
        }
        mma_commit(&bar);
    }
    __syncwarp();
    if (!mbar_wait(&bar, 0)) {
        if ((tid & 31) == 0) atomicExch(err, 1);
    }
    tc_fence_after();
    // dump all 128 lanes x N columns
    for (int col = 0; col < c.N; col += 32) {
        uint32_t r[32];
        tmem_ld32(tmem_addr(tm, warp * 32, col), r);
        tmem_wait_ld();
        const int lane = warp * 32 + (tid & 31);
        for (int j = 0; j < 32 && col + j < c.N; ++j)
            D[lane * c.N + col + j] = __uint_as_float(r[j]);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tm, 256);
        tmem_relinquish();
    }
}

extern "C" int umma_probe(int M, int N, int K, int a_mn, int b_mn, int b_swz, int neg_a,
                          int a_tmem, const uint16_t *A_h, const uint16_t *B_h, float *D_h) {
    if (M * K * 2 > 32768 || K * N * 2 > 32768 || N % 32 != 0 || N > 256) return -1;
    if (a_tmem && (M != 128 || N > 128 || K % 32 != 0 || K > 128 || a_mn)) return -1;
    ProbeCfg c{M, N, K, a_mn, b_mn, b_swz, neg_a, a_tmem};
    uint16_t *A, *B;
    float *D;
    int *err;
    if (cudaMalloc(&A, M * K * 2) || cudaMalloc(&B, K * N * 2) || cudaMalloc(&D, 128 * N * 4) ||
        cudaMalloc(&err, 4))
        return -2;
    cudaMemcpy(A, A_h, M * K * 2, cudaMemcpyHostToDevice);
    cudaMemcpy(B, B_h, K * N * 2, cudaMemcpyHostToDevice);
    cudaMemset(D, 0, 128 * N * 4);
    cudaMemset(err, 0, 4);
    cudaFuncSetAttribute(probe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 65536 + 1024);
    probe_kernel<<<1, 128, 65536 + 1024>>>(c, A, B, D, err);
    cudaError_t e = cudaDeviceSynchronize();
    int herr = 0;
    cudaMemcpy(D_h, D, 128 * N * 4, cudaMemcpyDeviceToHost);
    cudaMemcpy(&herr, err, 4, cudaMemcpyDeviceToHost);
    cudaFree(A); cudaFree(B); cudaFree(D); cudaFree(err);
    if (e != cudaSuccess) return -3;
    return herr ? -4 : 0;
}
