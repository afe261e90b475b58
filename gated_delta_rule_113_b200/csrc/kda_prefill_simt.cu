// kda_prefill_simt.cu -- chunked KDA prefill on CUDA cores, fp32 throughout.
//
// This is the fp32-accurate path (fp32 I/O needs ~1e-4 relative accuracy,
// beyond bf16/tf32 tensor-core operands).  It evaluates the recurrence of
// the page "Kimi K3: Open Frontier Intelligence and Implementation
// Framework" (section "Hybrid Attention Mechanism", KDA bullet: delta rule
// with a channel-wise forget gate)
//     S_t = (I - b_t k_t k_t^T) Diag(a_t) S_{t-1} + b_t k_t v_t^T,  o_t = S_t^T q_t
// 64 tokens at a time.  Per chunk of L <= 64 rows entering with state S
// (g = in-chunk inclusive cumsum of log a per channel, Gam = exp(g)):
//     Qg = Q*Gam, Kg = K*Gam, Ki = K/Gam                  (row-wise, per channel)
//     A  = strict_lower(diag(b) Kg Ki^T),  Tb = (I + A)^{-1} diag(b)
//     U  = Tb (V - Kg S)
//     O  = Qg S + lower_incl(Qg Ki^T) U
//     S' = Diag(Gam_L) (S + Ki^T U)
// Rows past the end of a sequence are zero with log a = 0, which leaves
// every quantity above unchanged for the valid rows.
//
// Work decomposition: one CTA per (sequence, head, 32-wide slice of d_v).
// Every step after A is separable over the columns of V, so slices of one
// chain are independent; the slice CTAs recompute the key-side tiles.
// Sequences are visited longest-first (order from the varlen index).
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kThreads = 256;
constexpr int kVs = 32;  // d_v columns per CTA

// C[M][N] = sum_kk a(m, kk) * b(kk, n), each of the 256 threads owning a
// (M/16) x (N/16) register tile with rows ty + 16 i and columns tx + 16 j.
template <int M, int N, int KD, class FA, class FB, class FO>
__device__ __forceinline__ void tile_gemm(const FA &a, const FB &b, const FO &o) {
    constexpr int RM = M / 16, RN = N / 16;
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
    float acc[RM][RN];
#pragma unroll
    for (int i = 0; i < RM; ++i)
#pragma unroll
        for (int j = 0; j < RN; ++j) acc[i][j] = 0.f;
#pragma unroll 4
    for (int kk = 0; kk < KD; ++kk) {
        float av[RM], bv[RN];
#pragma unroll
        for (int i = 0; i < RM; ++i) av[i] = a(ty + 16 * i, kk);
#pragma unroll
        for (int j = 0; j < RN; ++j) bv[j] = b(kk, tx + 16 * j);
#pragma unroll
        for (int i = 0; i < RM; ++i)
#pragma unroll
            for (int j = 0; j < RN; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
#pragma unroll
    for (int i = 0; i < RM; ++i)
#pragma unroll
        for (int j = 0; j < RN; ++j) o(ty + 16 * i, tx + 16 * j, acc[i][j]);
}

template <int DK>
struct Smem {
    static constexpr int LDK = DK + 1;   // padded row strides (bank spread)
    static constexpr int LDC = kChunk + 1;
    static constexpr int LDV = kVs + 1;
    float Qg[kChunk * LDK];
    float Kg[kChunk * LDK];
    float Ki[kChunk * LDK];
    float A[kChunk * LDC];
    float P[kChunk * LDC];
    float Tb[kChunk * LDC];
    float X[kChunk * LDV];
    float U[kChunk * LDV];
    float S[DK * LDV];
    float b[kChunk];
    float gl[DK];
};

template <typename TIO, typename TG, int DK>
__global__ void __launch_bounds__(kThreads)
prefill_simt_kernel(const TIO *__restrict__ q, const TIO *__restrict__ k,
                    const TIO *__restrict__ v, const TG *__restrict__ la,
                    const TG *__restrict__ beta, const float *__restrict__ S0,
                    const int32_t *__restrict__ cu, TIO *__restrict__ out,
                    float *__restrict__ Sf, const int32_t *__restrict__ order, int N, int T,
                    int H, int Dv, int32_t *status) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    Smem<DK> &sm = *reinterpret_cast<Smem<DK> *>(smem_raw);
    constexpr int LDK = Smem<DK>::LDK, LDC = Smem<DK>::LDC, LDV = Smem<DK>::LDV;

    const int n_slices = Dv / kVs;
    const int per_seq = H * n_slices;
    const int n = order[blockIdx.x / per_seq];
    const int h = (blockIdx.x % per_seq) / n_slices;
    const int vs = blockIdx.x % n_slices;
    const int tid = threadIdx.x;

    int t0, t1;
    if (!seq_range(cu, n, T, t0, t1)) {
        set_status(status, KDA_ERR_SEQLENS);
        return;
    }

    // initial state slice S[c][j] = S0[n, h, c, vs*32 + j]
    const size_t sbase = ((size_t)n * H + h) * DK * Dv + (size_t)vs * kVs;
    for (int i = tid; i < DK * kVs; i += kThreads) {
        const int c = i / kVs, j = i % kVs;
        sm.S[c * LDV + j] = S0 ? S0[sbase + (size_t)c * Dv + j] : 0.f;
    }

    for (int c0 = t0; c0 < t1; c0 += kChunk) {
        const int L = min(kChunk, t1 - c0);
        __syncthreads();  // previous chunk fully consumed

        // ---- gates, scaled operands: one thread per key channel ----------
        // exp(g) and exp(-g) stay in fp32 range while the in-chunk cumulative
        // log-decay g is in [-80, 0]; a log_alpha above 0 or not finite, or a
        // g below -80, records KDA_ERR_DECAY (this chain's results are then
        // unspecified, nothing is read or written out of range).
        if (tid < DK) {
            const int c = tid;
            float g = 0.f;
            bool bad = false;
            for (int r = 0; r < kChunk; ++r) {
                float qg = 0.f, kg = 0.f, ki = 0.f;
                if (r < L) {
                    const size_t row = ((size_t)(c0 + r) * H + h) * DK + c;
                    const float lav = to_f32(la[row]);
                    bad |= !(lav <= 0.f);
                    g += lav;
                    const float kv = to_f32(k[row]);
                    const float e = expf(g);
                    qg = to_f32(q[row]) * e;
                    kg = kv * e;
                    ki = kv * expf(-g);
                }
                sm.Qg[r * LDK + c] = qg;
                sm.Kg[r * LDK + c] = kg;
                sm.Ki[r * LDK + c] = ki;
            }
            sm.gl[c] = expf(g);
            bad |= !(g >= -80.f);
            if (bad) set_status(status, KDA_ERR_DECAY);
        } else {
            for (int i = tid - DK; i < kChunk * kVs; i += kThreads - DK) {
                const int r = i / kVs, j = i % kVs;
                sm.X[r * LDV + j] =
                    r < L ? to_f32(v[((size_t)(c0 + r) * H + h) * Dv + vs * kVs + j]) : 0.f;
            }
            for (int r = tid - DK; r < kChunk; r += kThreads - DK)
                sm.b[r] = r < L ? to_f32(beta[(size_t)(c0 + r) * H + h]) : 0.f;
        }
        __syncthreads();

        // ---- A = strict_lower(diag(b) Kg Ki^T), P = lower_incl(Qg Ki^T) ----
        {
            constexpr int RM = 4, RN = 4;
            const int tx = tid % 16, ty = tid / 16;
            float aa[RM][RN], pp[RM][RN];
#pragma unroll
            for (int i = 0; i < RM; ++i)
#pragma unroll
                for (int j = 0; j < RN; ++j) aa[i][j] = pp[i][j] = 0.f;
#pragma unroll 4
            for (int c = 0; c < DK; ++c) {
                float kv[RM], qv[RM], iv[RN];
#pragma unroll
                for (int i = 0; i < RM; ++i) {
                    kv[i] = sm.Kg[(ty + 16 * i) * LDK + c];
                    qv[i] = sm.Qg[(ty + 16 * i) * LDK + c];
                }
#pragma unroll
                for (int j = 0; j < RN; ++j) iv[j] = sm.Ki[(tx + 16 * j) * LDK + c];
#pragma unroll
                for (int i = 0; i < RM; ++i)
#pragma unroll
                    for (int j = 0; j < RN; ++j) {
                        aa[i][j] = fmaf(kv[i], iv[j], aa[i][j]);
                        pp[i][j] = fmaf(qv[i], iv[j], pp[i][j]);
                    }
            }
#pragma unroll
            for (int i = 0; i < RM; ++i)
#pragma unroll
                for (int j = 0; j < RN; ++j) {
                    const int r = ty + 16 * i, s = tx + 16 * j;
                    sm.A[r * LDC + s] = s < r ? sm.b[r] * aa[i][j] : 0.f;
                    sm.P[r * LDC + s] = s <= r ? pp[i][j] : 0.f;
                }
        }
        __syncthreads();

        // ---- Tb = (I + A)^{-1} diag(b): forward substitution, one column per
        //      thread; seeding the diagonal with b_j scales column j by b_j.
        if (tid < kChunk) {
            const int j = tid;
            for (int i = 0; i < kChunk; ++i) {
                float t;
                if (i < j) {
                    t = 0.f;
                } else if (i == j) {
                    t = sm.b[j];
                } else {
                    float s = 0.f;
                    for (int m = j; m < i; ++m) s = fmaf(sm.A[i * LDC + m], sm.Tb[m * LDC + j], s);
                    t = -s;
                }
                sm.Tb[i * LDC + j] = t;
            }
        }
        __syncthreads();

        // ---- X = V - Kg S ---------------------------------------------------
        tile_gemm<kChunk, kVs, DK>(
            [&](int r, int c) { return sm.Kg[r * LDK + c]; },
            [&](int c, int j) { return sm.S[c * LDV + j]; },
            [&](int r, int j, float acc) { sm.X[r * LDV + j] -= acc; });
        __syncthreads();

        // ---- U = Tb X -------------------------------------------------------
        tile_gemm<kChunk, kVs, kChunk>(
            [&](int r, int s) { return sm.Tb[r * LDC + s]; },
            [&](int s, int j) { return sm.X[s * LDV + j]; },
            [&](int r, int j, float acc) { sm.U[r * LDV + j] = acc; });
        __syncthreads();

        // ---- O = Qg S + P U -> out ------------------------------------------
        tile_gemm<kChunk, kVs, DK + kChunk>(
            [&](int r, int kk) {
                return kk < DK ? sm.Qg[r * LDK + kk] : sm.P[r * LDC + (kk - DK)];
            },
            [&](int kk, int j) { return kk < DK ? sm.S[kk * LDV + j] : sm.U[(kk - DK) * LDV + j]; },
            [&](int r, int j, float acc) {
                if (r < L) out[((size_t)(c0 + r) * H + h) * Dv + vs * kVs + j] = from_f32<TIO>(acc);
            });
        __syncthreads();

        // ---- S <- Diag(Gam_L) (S + Ki^T U) ----------------------------------
        tile_gemm<DK, kVs, kChunk>(
            [&](int c, int s) { return sm.Ki[s * LDK + c]; },
            [&](int s, int j) { return sm.U[s * LDV + j]; },
            [&](int c, int j, float acc) {
                sm.S[c * LDV + j] = sm.gl[c] * (sm.S[c * LDV + j] + acc);
            });
    }
    __syncthreads();
    if (Sf) {
        for (int i = tid; i < DK * kVs; i += kThreads) {
            const int c = i / kVs, j = i % kVs;
            Sf[sbase + (size_t)c * Dv + j] = sm.S[c * LDV + j];
        }
    }
}

template <typename TIO, typename TG, int DK>
cudaError_t launch_typed(const ForwardArgs &a, cudaStream_t s) {
    auto kern = prefill_simt_kernel<TIO, TG, DK>;
    const int smem = (int)sizeof(Smem<DK>);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)a.N * a.H * (a.Dv / kVs);
    kern<<<grid, kThreads, smem, s>>>(
        (const TIO *)a.q, (const TIO *)a.k, (const TIO *)a.v, (const TG *)a.log_alpha,
        (const TG *)a.beta, a.S0, a.cu_seqlens, (TIO *)a.out, a.S_final, a.order, a.N, a.T, a.H,
        a.Dv, a.status);
    return cudaGetLastError();
}

template <typename TIO, typename TG>
cudaError_t launch_dk(const ForwardArgs &a, cudaStream_t s) {
    return a.Dk == 64 ? launch_typed<TIO, TG, 64>(a, s) : launch_typed<TIO, TG, 128>(a, s);
}

}  // namespace

cudaError_t launch_prefill_simt(const ForwardArgs &a, cudaStream_t s) {
    const bool io16 = a.io_dtype == KDA_BF16, g16 = a.gate_dtype == KDA_BF16;
    if (io16 && g16) return launch_dk<__nv_bfloat16, __nv_bfloat16>(a, s);
    if (io16) return launch_dk<__nv_bfloat16, float>(a, s);
    if (g16) return launch_dk<float, __nv_bfloat16>(a, s);
    return launch_dk<float, float>(a, s);
}

}  // namespace kda
