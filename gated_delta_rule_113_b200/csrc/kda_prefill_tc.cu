// kda_prefill_tc.cu -- chunked KDA prefill on the sm_100a tensor cores.
//
// The page "Kimi K3: Open Frontier Intelligence and Implementation Framework"
// (section "Hybrid Attention Mechanism", KDA bullet) notes that KDA's
// lower-bounded, channel-wise decay lets the diagonal (intra-chunk) and
// off-diagonal (inter-chunk) tiles of a chunked evaluation run as dense
// tensor-core products.  This kernel does exactly that for bf16 inputs with
// an fp32 state.  Per chunk of 64 tokens entering with state S (g = in-chunk
// inclusive cumsum of log alpha per channel, Gam = exp(g)):
//
//   prep   Qg = Q*Gam, Kg = K*Gam, Ki = K/Gam, Gam_L             CUDA cores
//   MMA_AP [A; P] = [Kg; Qg] Ki^T          (M=128, N=64, K=128)   tcgen05
//   solve  Tb = (I + strict(diag(b) A))^{-1} diag(b)              CUDA cores +
//          P  = lower_incl(P)                                      mma.sync tf32
//   MMA_W  W  = Tb Kg                      (M=128 padded, N=128, K=64)
//   MMA_0  D1 = Tb V          (= U0)       (M=128 padded, N=VS, K=64)
//   MMA_1  D1 += [-W; Qg] S   (U rows 0-63, Qg S rows 64-127; K=128)   chain
//   MMA_2  dS = Ki^T U                     (M=128, N=VS, K=64)         chain
//   MMA_3  D1 += [0; P] U     (rows 64-127 become O)
//   state  S <- Diag(Gam_L) (S + dS)       fp32, in registers          chain
//
// The decay products Gam (and 1/Gam) come from running products of
// alpha = 2^(log_alpha * log2 e) inside the chunk, so each gate element costs
// one exponential; the scaled operands are formed with packed bf16 products.
//
// One CTA owns one (sequence, head, VS-wide slice of d_v): everything after
// MMA_W is separable over value columns.  Warp roles (19 warps):
//   0-3    chain: thread c owns state row c (fp32 registers); warps 0-1 turn
//          U into the bf16 operand, warps 2-3 write the outputs
//   4-11   prep: gates and the scaled operands, in place over the TMA tiles
//   12-15  solve: triangular inverse, P mask, W -> bf16 operand
//   16     TMA producer
//   17     key-side MMA issuer (MMA_AP, MMA_W, MMA_0); owns TMEM
//   18     chain MMA issuer (MMA_1, MMA_2, MMA_3)
// Two pipeline stages of operand tiles let the key-side work of chunk n+1
// overlap the sequential state chain of chunk n.  All waits are bounded.
#include <cuda.h>

#include "kda_internal.cuh"
#include "kda_tc_common.cuh"
#include "sm100.cuh"

namespace kda {
namespace {

using namespace sm100;
using namespace tc;

// Optional per-chunk timeline of CTA 0 (clock64 per pipeline event), compiled
// in only with -DKDA_TRACE for profiling builds; a no-op otherwise.
#ifdef KDA_TRACE
__device__ unsigned long long g_kda_trace[64 * 32];
#define KDA_TRACE_EVENT(n, e)                                                    \
    do {                                                                         \
        if (blockIdx.x == 0 && (n) < 64) g_kda_trace[(n) * 32 + (e)] = clock64(); \
    } while (0)
#else
#define KDA_TRACE_EVENT(n, e) \
    do {                      \
    } while (0)
#endif

constexpr int kWarps = 19;
constexpr int kThreads = kWarps * 32;

enum Role { kChain0 = 0, kPrep0 = 4, kSolve0 = 12, kTma = 16, kMmaK = 17, kMmaC = 18 };
enum NamedBar { kBarPrep = 1, kBarSolve = 2 };

template <int VS>
struct Layout {
    // shared-memory byte offsets (relative to a 1024-aligned base)
    static constexpr uint32_t kKQ = 0;                      // 2 x 32 KB: [katom][Kg|Qg rows]
    static constexpr uint32_t kKI = kKQ + 2 * 32768;        // 2 x 16 KB: [katom][64 rows]
    static constexpr uint32_t kTP = kKI + 2 * 16384;        // 2 x 24 KB: Tb | 0 | P
    static constexpr uint32_t kVsz = 64 * VS * 2;
    static constexpr uint32_t kV = kTP + 2 * 24576;         // 2 x V tile
    static constexpr uint32_t kSB = kV + 2 * kVsz;          // bf16 state operand
    static constexpr uint32_t kUB = kSB + 128 * VS * 2;     // bf16 U operand
    static constexpr uint32_t kL = kUB + 64 * VS * 2;       // fp32 [64][kLDL]
    static constexpr uint32_t kT = kL + 64 * kLDL * 4;      // fp32 [64][kLDL]
    static constexpr uint32_t kGP = kT + 64 * kLDL * 4;     // fp32 [16][128] group products / prefix
    static constexpr uint32_t kSUF = kGP + 16 * 128 * 4;    // fp32 [16][128] suffix
    static constexpr uint32_t kGL = kSUF + 16 * 128 * 4;    // fp32 [2][128]
    static constexpr uint32_t kB = kGL + 2 * 128 * 4;       // fp32 [2][64]
    static constexpr uint32_t kBar = kB + 2 * 64 * 4;       // mbarriers
    static constexpr uint32_t kNumBars = 32;
    static constexpr uint32_t kMisc = kBar + kNumBars * 8;  // tmem base, abort flag
    static constexpr uint32_t kSize = kMisc + 16;
    static constexpr uint32_t kAlloc = kSize + 1024;        // + alignment slack
    static_assert(kAlloc <= 232448, "shared memory budget exceeded");
    static_assert(VS == 32, "value slice width");

    // TMEM columns
    static constexpr uint32_t kTmAP = 0;
    static constexpr uint32_t kTmW = 64;
    static constexpr uint32_t kTmD1 = 192;       // + s * VS
    static constexpr uint32_t kTmD2 = 192 + 2 * VS;
    static constexpr uint32_t kTmCols = 512;
};

// mbarrier indices
enum Bars {
    bRawFull = 0,    // [2] TMA -> prep (tx bytes)
    bKqFull = 2,     // [2] prep -> key-side issuer, chain warps
    bApFull = 4,     // MMA_AP done -> solve
    bApFree = 5,     // solve read D_AP -> key-side issuer
    bTbFull = 6,     // [2] solve wrote Tb, P -> key-side issuer
    bWaccFull = 8,   // MMA_W done -> solve
    bWReady = 9,     // [2] -W operand written -> chain issuer (and D_W free)
    bU0Done = 11,    // [2] MMA_0 done -> chain issuer
    bSbFull = 13,    // chain warps wrote bf16 S -> chain issuer
    bUFull = 14,     // MMA_1 done -> chain warps 0-1
    bUbFull = 15,    // bf16 U written -> chain issuer
    bDsFull = 16,    // MMA_2 done -> chain warps
    bOFull = 17,     // [2] MMA_3 done -> output warps
    bD1Free = 19,    // [2] output read D1 -> key-side issuer
    bStageFree = 21, // [2] every MMA of a stage done -> TMA producer
    bDrainK = 23,    // issuers drain before exit
    bDrainC = 24,
    bNum = 25
};

struct TcParams {
    const __nv_bfloat16 *beta;
    const float *S0;
    const int32_t *cu;
    __nv_bfloat16 *out;
    float *Sf;
    const int32_t *order;
    int32_t *status;
    int N, T, H;
};


template <int VS>
__global__ void __launch_bounds__(kThreads, 1)
prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_la,
                  const __grid_constant__ CUtensorMap tm_v, TcParams p) {
    using Ly = Layout<VS>;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    // align by offsetting the shared array itself, so every derived pointer
    // stays a known shared-memory address (ld.shared, not generic loads)
    unsigned char *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(sm);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + Ly::kBar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + Ly::kMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + Ly::kMisc + 4);
    float *sL = reinterpret_cast<float *>(sm + Ly::kL);
    float *sT = reinterpret_cast<float *>(sm + Ly::kT);
    float *sGP = reinterpret_cast<float *>(sm + Ly::kGP);
    float *sSUF = reinterpret_cast<float *>(sm + Ly::kSUF);
    float *sGL = reinterpret_cast<float *>(sm + Ly::kGL);
    float *sB = reinterpret_cast<float *>(sm + Ly::kB);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n_slices = kDV / VS;
    const int per_seq = p.H * n_slices;
    const int seq = p.order[blockIdx.x / per_seq];
    const int h = (blockIdx.x % per_seq) / n_slices;
    const int vs = blockIdx.x % n_slices;
    int t0, t1;
    if (!seq_range(p.cu, seq, p.T, t0, t1)) {
        if (tid == 0) set_status(p.status, KDA_ERR_SEQLENS);
        return;
    }
    const int nchunks = (t1 - t0 + kChunk - 1) / kChunk;
    const size_t sbase_g = ((size_t)seq * p.H + h) * kDK * kDV + (size_t)vs * VS;

    // ---------------------------------------------------------------- setup
    if (tid == 0) {
        for (int i = 0; i < bNum; ++i) {
            uint32_t cnt = 1;
            if (i == bKqFull || i == bKqFull + 1) cnt = kPrepThreads / 32;
            if (i == bWReady || i == bWReady + 1) cnt = 2;
            if (i == bSbFull) cnt = 4;
            if (i == bUbFull) cnt = 2;
            if (i == bD1Free || i == bD1Free + 1) cnt = 2;
            mbar_init(&bars[i], cnt);
        }
        abort_flag[0] = 0;
        abort_flag[1] = 0;
        fence_mbar_init();
    }
    if (warp == kTma && lane == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_la);
        prefetch_tmap(&tm_v);
    }
    // rows 64..127 of both Tb|0|P tiles stay zero (never written afterwards)
    for (int i = tid; i < 2 * 512; i += kThreads) {
        const int s = i / 512, j = i % 512;
        sts128(sbase + Ly::kTP + s * 24576 + 8192 + j * 16, 0, 0, 0, 0);
    }
    // blocks of T above the 16x16 diagonal blocks stay zero; the solve only
    // ever writes the lower blocks
    for (int i = tid; i < 64 * kLDL / 4; i += kThreads)
        sts128(sbase + Ly::kT + i * 16, 0, 0, 0, 0);
    if (warp == kMmaK) {
        tmem_alloc(tmem_slot, Ly::kTmCols);
        tmem_relinquish();
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // ================================================================ roles
    if (warp == kTma) {
        // ---------------------------------------------------- TMA producer
        if (lane == 0) {
            for (int n = 0; n < nchunks; ++n) {
                const int s = n & 1;
                if (n >= 2 && !wait_or_abort(&bars[bStageFree + s], ((n - 2) >> 1) & 1, abort_flag,
                                             p.status))
                    break;
                const int c0 = t0 + n * kChunk;
                uint64_t *full = &bars[bRawFull + s];
                mbar_arrive_expect_tx(full, 6 * 8192 + 64 * VS * 2);
                for (int a = 0; a < 2; ++a) {
                    tma_load_3d(sm + Ly::kKQ + s * 32768 + a * 16384, &tm_k, full, a * 64, h, c0);
                    tma_load_3d(sm + Ly::kKQ + s * 32768 + a * 16384 + 8192, &tm_q, full, a * 64, h,
                                c0);
                    tma_load_3d(sm + Ly::kKI + s * 16384 + a * 8192, &tm_la, full, a * 64, h, c0);
                }
                tma_load_3d(sm + Ly::kV + s * Ly::kVsz, &tm_v, full, vs * VS, h, c0);
                KDA_TRACE_EVENT(n, 0);
                if (n + 2 < nchunks) {
                    const int c2 = c0 + 2 * kChunk;
                    for (int a = 0; a < 2; ++a) {
                        tma_prefetch_3d(&tm_k, a * 64, h, c2);
                        tma_prefetch_3d(&tm_q, a * 64, h, c2);
                        tma_prefetch_3d(&tm_la, a * 64, h, c2);
                    }
                    tma_prefetch_3d(&tm_v, vs * VS, h, c2);
                }
            }
            // every armed load must land before the CTA may exit
            for (int n = max(0, nchunks - 2); n < nchunks; ++n)
                mbar_wait(&bars[bRawFull + (n & 1)], (n >> 1) & 1);
        }
    } else if (warp >= kPrep0 && warp < kPrep0 + kPrepThreads / 32) {
        // ----------------------------------------------------------- prep
        // thread = (row group rg of 4 rows, channel group cg of 8 channels)
        const int t = tid - kPrep0 * 32;
        for (int n = 0; n < nchunks; ++n) {
            const int s = n & 1;
            const int c0 = t0 + n * kChunk;
            const int L = min(kChunk, t1 - c0);
            if (!wait_or_abort(&bars[bRawFull + s], (n >> 1) & 1, abort_flag, p.status)) break;
            if (t == 0) KDA_TRACE_EVENT(n, 1);
            prep_chunk(t, sbase + Ly::kKQ + s * 32768, sbase + Ly::kKI + s * 16384, sGP, sSUF,
                       sGL + s * 128, sB + s * 64, p.beta, c0, L, p.H, h, kBarPrep, p.status);
            __syncwarp();
            if (t == 0) KDA_TRACE_EVENT(n, 2);
            if (lane == 0) mbar_arrive(&bars[bKqFull + s]);
        }
    } else if (warp >= kSolve0 && warp < kSolve0 + 4) {
        // ---------------------------------------------------------- solve
        const int sw = warp - kSolve0;        // 0..3, TMEM lanes 32*sw..
        const int t = tid - kSolve0 * 32;     // 0..127
        for (int n = 0; n < nchunks; ++n) {
            const int s = n & 1;
            if (!wait_or_abort(&bars[bApFull], n & 1, abort_flag, p.status)) break;
            tc_fence_after();
            if (t == 0) KDA_TRACE_EVENT(n, 4);
            solve_chunk(sw, lane, tmem, Ly::kTmAP, sbase + Ly::kTP + s * 24576 + 16384, sL, sT,
                        sB + s * 64, &bars[bApFree], kBarSolve);
            write_tb(sw, lane, sbase + Ly::kTP + s * 24576, sT, sB + s * 64, kBarSolve);
            if (t == 0) mbar_arrive(&bars[bTbFull + s]);
            if (t == 0) KDA_TRACE_EVENT(n, 9);

            // W = Tb Kg (TMEM, fp32) -> -W as bf16 over the Kg rows of this stage
            if (sw < 2) {
                if (!wait_or_abort(&bars[bWaccFull], n & 1, abort_flag, p.status)) break;
                tc_fence_after();
                if (t == 0) KDA_TRACE_EVENT(n, 11);
                convert_w(sw, lane, tmem, Ly::kTmW, sbase + Ly::kKQ + s * 32768);
                if (lane == 0) mbar_arrive(&bars[bWReady + s]);
                if (t == 0) KDA_TRACE_EVENT(n, 12);
            }
        }
    } else if (warp == kMmaK) {
        // --------------------------------------------- key-side MMA issuer
        if (lane == 0) {
            constexpr uint32_t kIdAP = idesc_bf16(128, 64, 0, 0);
            constexpr uint32_t kIdW = idesc_bf16(128, 128, 0, 1);
            constexpr uint32_t kIdV = idesc_bf16(128, VS, 0, 1);
            for (int n = 0; n < nchunks; ++n) {
                const int s = n & 1;
                const uint32_t kq = sbase + Ly::kKQ + s * 32768;
                const uint32_t ki = sbase + Ly::kKI + s * 16384;
                const uint32_t tp = sbase + Ly::kTP + s * 24576;
                const uint32_t vt = sbase + Ly::kV + s * Ly::kVsz;
                const uint64_t d_kq = smem_desc(kq, 16, 1024, kSw128);
                const uint64_t d_ki = smem_desc(ki, 16, 1024, kSw128);
                const uint64_t d_tp = smem_desc(tp, 16, 1024, kSw128);
                const uint64_t d_kg = smem_desc(kq, 16384, 1024, kSw128);
                const uint64_t d_v = vs_desc<VS>(vt, 64);
                if (!wait_or_abort(&bars[bKqFull + s], (n >> 1) & 1, abort_flag, p.status)) break;
                if (n >= 1 && !wait_or_abort(&bars[bApFree], (n - 1) & 1, abort_flag, p.status)) break;
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_bf16(tmem + Ly::kTmAP, d_kq + kmaj_step(ks, 16384), d_ki + kmaj_step(ks, 8192),
                             kIdAP, ks > 0);
                mma_commit(&bars[bApFull]);
                KDA_TRACE_EVENT(n, 3);

                if (!wait_or_abort(&bars[bTbFull + s], (n >> 1) & 1, abort_flag, p.status)) break;
                if (n >= 1 && !wait_or_abort(&bars[bWReady + ((n - 1) & 1)], ((n - 1) >> 1) & 1,
                                             abort_flag, p.status))
                    break;
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tmem + Ly::kTmW, d_tp + ((uint64_t)(ks * 32) >> 4),
                             d_kg + ((uint64_t)(ks * 2048) >> 4), kIdW, ks > 0);
                mma_commit(&bars[bWaccFull]);
                KDA_TRACE_EVENT(n, 10);

                if (n >= 2 && !wait_or_abort(&bars[bD1Free + s], ((n - 2) >> 1) & 1, abort_flag,
                                             p.status))
                    break;
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tmem + Ly::kTmD1 + s * VS, d_tp + ((uint64_t)(ks * 32) >> 4),
                             d_v + vs_step<VS>(ks), kIdV, ks > 0);
                mma_commit(&bars[bU0Done + s]);
                KDA_TRACE_EVENT(n, 13);
            }
            mma_commit(&bars[bDrainK]);
            mbar_wait(&bars[bDrainK], 0);
        }
    } else if (warp == kMmaC) {
        // ------------------------------------------------- chain MMA issuer
        if (lane == 0) {
            constexpr uint32_t kIdV = idesc_bf16(128, VS, 0, 1);
            constexpr uint32_t kIdS = idesc_bf16(128, VS, 1, 1);
            const uint64_t d_sb = vs_desc<VS>(sbase + Ly::kSB, 128);
            const uint64_t d_ub = vs_desc<VS>(sbase + Ly::kUB, 64);
            for (int n = 0; n < nchunks; ++n) {
                const int s = n & 1;
                const uint32_t kq = sbase + Ly::kKQ + s * 32768;
                const uint32_t ki = sbase + Ly::kKI + s * 16384;
                const uint32_t tp = sbase + Ly::kTP + s * 24576;
                const uint32_t d1 = tmem + Ly::kTmD1 + s * VS;
                const uint64_t d_kq = smem_desc(kq, 16, 1024, kSw128);
                const uint64_t d_kit = smem_desc(ki, 8192, 1024, kSw128);
                const uint64_t d_p = smem_desc(tp + 8192, 16, 1024, kSw128);
                if (!wait_or_abort(&bars[bWReady + s], (n >> 1) & 1, abort_flag, p.status)) break;
                KDA_TRACE_EVENT(n, 21);
                if (!wait_or_abort(&bars[bU0Done + s], (n >> 1) & 1, abort_flag, p.status)) break;
                KDA_TRACE_EVENT(n, 22);
                if (!wait_or_abort(&bars[bSbFull], n & 1, abort_flag, p.status)) break;
                KDA_TRACE_EVENT(n, 23);
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_bf16(d1, d_kq + kmaj_step(ks, 16384), d_sb + vs_step<VS>(ks), kIdV, 1);
                mma_commit(&bars[bUFull]);
                KDA_TRACE_EVENT(n, 14);
                if (!wait_or_abort(&bars[bUbFull], n & 1, abort_flag, p.status)) break;
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tmem + Ly::kTmD2, d_kit + ((uint64_t)(ks * 2048) >> 4),
                             d_ub + vs_step<VS>(ks), kIdS, ks > 0);
                mma_commit(&bars[bDsFull]);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(d1, d_p + ((uint64_t)(ks * 32) >> 4), d_ub + vs_step<VS>(ks), kIdV, 1);
                mma_commit(&bars[bOFull + s]);
                mma_commit(&bars[bStageFree + s]);
                KDA_TRACE_EVENT(n, 17);
            }
            mma_commit(&bars[bDrainC]);
            mbar_wait(&bars[bDrainC], 0);
        }
    } else if (warp < kChain0 + 4) {
        // ------------------------------------------------------ chain warps
        const int c = tid;                 // state row (key channel) 0..127
        const int wq = warp;               // TMEM lane quarter
        float S[VS];
        {
            const float *src = p.S0 ? p.S0 + sbase_g + (size_t)c * kDV : nullptr;
#pragma unroll
            for (int j = 0; j < VS; j += 4) {
                float4 v = src ? *reinterpret_cast<const float4 *>(src + j) : make_float4(0, 0, 0, 0);
                S[j] = v.x; S[j + 1] = v.y; S[j + 2] = v.z; S[j + 3] = v.w;
            }
        }
        auto store_out = [&](int m) {
            // outputs of chunk m: D1 lanes 64..127 hold O rows 0..63
            const int sm1 = m & 1;
            const int c0 = t0 + m * kChunk, L = min(kChunk, t1 - c0);
            const int r = c - 64;
#pragma unroll
            for (int j = 0; j < VS; j += 32) {
                uint32_t v[32];
                tmem_ld32(tmem_addr(tmem, 32 * wq, Ly::kTmD1 + sm1 * VS + j), v);
                tmem_wait_ld();
                if (r < L) {
                    __nv_bfloat16 *dst = p.out + ((size_t)(c0 + r) * p.H + h) * kDV + vs * VS + j;
#pragma unroll
                    for (int e = 0; e < 32; e += 8) {
                        uint4 w;
                        w.x = pack2(__uint_as_float(v[e]), __uint_as_float(v[e + 1]));
                        w.y = pack2(__uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
                        w.z = pack2(__uint_as_float(v[e + 4]), __uint_as_float(v[e + 5]));
                        w.w = pack2(__uint_as_float(v[e + 6]), __uint_as_float(v[e + 7]));
                        *reinterpret_cast<uint4 *>(dst + e) = w;
                    }
                }
            }
        };
        float gl_cur = 1.f;
        bool ok = true;
        for (int n = 0; n <= nchunks && ok; ++n) {
            if (n > 0) {
                // S <- Diag(Gam_L) (S + dS) for chunk n-1
                if (!wait_or_abort(&bars[bDsFull], (n - 1) & 1, abort_flag, p.status)) { ok = false; break; }
                tc_fence_after();
                if (c == 0) KDA_TRACE_EVENT(n - 1, 18);
#pragma unroll
                for (int j = 0; j < VS; j += 32) {
                    uint32_t v[32];
                    tmem_ld32(tmem_addr(tmem, 32 * wq, Ly::kTmD2 + j), v);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) S[j + e] = gl_cur * (S[j + e] + __uint_as_float(v[e]));
                }
            }
            if (n == nchunks) {
                if (wq >= 2 && n > 0) {
                    const int m = n - 1;
                    if (!wait_or_abort(&bars[bOFull + (m & 1)], (m >> 1) & 1, abort_flag, p.status)) { ok = false; break; }
                    tc_fence_after();
                    store_out(m);
                }
                break;
            }
            const int s = n & 1;
            // Gam_L of this chunk (prep done) and the bf16 state operand
            if (!wait_or_abort(&bars[bKqFull + s], (n >> 1) & 1, abort_flag, p.status)) { ok = false; break; }
            gl_cur = sGL[s * 128 + c];
            if (c == 0) KDA_TRACE_EVENT(n, 20);
            {
                const uint32_t sb = sbase + Ly::kSB;
#pragma unroll
                for (int j = 0; j < VS / 8; ++j) {
                    sts128(sb + vs_off<VS>(c, j), pack2(S[8 * j], S[8 * j + 1]),
                           pack2(S[8 * j + 2], S[8 * j + 3]), pack2(S[8 * j + 4], S[8 * j + 5]),
                           pack2(S[8 * j + 6], S[8 * j + 7]));
                }
            }
            fence_proxy_async();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[bSbFull]);
            if (c == 0) KDA_TRACE_EVENT(n, 19);

            if (wq < 2) {
                // U rows: D1 lanes 0..63 -> bf16 operand
                if (!wait_or_abort(&bars[bUFull], n & 1, abort_flag, p.status)) { ok = false; break; }
                tc_fence_after();
                if (c == 0) KDA_TRACE_EVENT(n, 15);
                const uint32_t ub = sbase + Ly::kUB;
#pragma unroll
                for (int j = 0; j < VS; j += 32) {
                    uint32_t v[32];
                    tmem_ld32(tmem_addr(tmem, 32 * wq, Ly::kTmD1 + s * VS + j), v);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; e += 8) {
                        sts128(ub + vs_off<VS>(c, (j + e) / 8),
                               pack2(__uint_as_float(v[e]), __uint_as_float(v[e + 1])),
                               pack2(__uint_as_float(v[e + 2]), __uint_as_float(v[e + 3])),
                               pack2(__uint_as_float(v[e + 4]), __uint_as_float(v[e + 5])),
                               pack2(__uint_as_float(v[e + 6]), __uint_as_float(v[e + 7])));
                    }
                }
                fence_proxy_async();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[bUbFull]);
                if (c == 0) KDA_TRACE_EVENT(n, 16);
            } else if (n > 0) {
                // outputs of chunk n-1
                const int m = n - 1;
                if (!wait_or_abort(&bars[bOFull + (m & 1)], (m >> 1) & 1, abort_flag, p.status)) { ok = false; break; }
                tc_fence_after();
                store_out(m);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[bD1Free + (m & 1)]);
            }
        }
        if (ok && p.Sf) {
            float *dst = p.Sf + sbase_g + (size_t)c * kDV;
#pragma unroll
            for (int j = 0; j < VS; j += 4)
                *reinterpret_cast<float4 *>(dst + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
        }
    }

    // ------------------------------------------------------------ teardown
    tc_fence_before();
    __syncthreads();
    if (tid == 0) report_abort(abort_flag, p.status);
    if (warp == kMmaK) {
        tc_fence_after();
        tmem_dealloc(tmem, Ly::kTmCols);
    }
}

template <int VS>
cudaError_t launch_vs(const ForwardArgs &a, cudaStream_t s) {
    CUtensorMap mq, mk, mla, mv;
    const int T = a.T > 0 ? a.T : 1;
    if (!make_tmap_bf16_3d(&mq, a.q, T, a.H, kDK, 64, 128) ||
        !make_tmap_bf16_3d(&mk, a.k, T, a.H, kDK, 64, 128) ||
        !make_tmap_bf16_3d(&mla, a.log_alpha, T, a.H, kDK, 64, 128) ||
        !make_tmap_bf16_3d(&mv, a.v, T, a.H, kDV, VS, VS * 2))
        return cudaErrorInvalidValue;
    TcParams p;
    p.beta = static_cast<const __nv_bfloat16 *>(a.beta);
    p.S0 = a.S0;
    p.cu = a.cu_seqlens;
    p.out = static_cast<__nv_bfloat16 *>(a.out);
    p.Sf = a.S_final;
    p.order = a.order;
    p.status = a.status;
    p.N = a.N;
    p.T = a.T;
    p.H = a.H;
    auto kern = prefill_tc_kernel<VS>;
    const int smem = (int)Layout<VS>::kAlloc;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)a.N * a.H * (kDV / VS);
    kern<<<grid, kThreads, smem, s>>>(mq, mk, mla, mv, p);
    return cudaGetLastError();
}

}  // namespace

bool prefill_tc_supported(const ForwardArgs &a) {
    return a.io_dtype == KDA_BF16 && a.gate_dtype == KDA_BF16 && a.Dk == tc::kDK &&
           a.Dv == tc::kDV;
}

cudaError_t launch_prefill_tc(const ForwardArgs &a, cudaStream_t s) {
    return launch_vs<32>(a, s);
}

}  // namespace kda

#ifdef KDA_TRACE
extern "C" int kda_trace_read(unsigned long long *host) {
    return (int)cudaMemcpyFromSymbol(host, kda::g_kda_trace, sizeof(kda::g_kda_trace));
}
#endif
