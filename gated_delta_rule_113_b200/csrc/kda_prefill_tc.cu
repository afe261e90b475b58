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
#include "sm100.cuh"

namespace kda {
namespace {

using namespace sm100;

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
constexpr int kDK = 128;           // key width handled by this kernel
constexpr int kDV = 128;           // value width handled by this kernel
constexpr int kLDL = 68;           // fp32 row stride of the solve scratch
constexpr int kPrepThreads = 256;

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
    static constexpr uint32_t kX = kT + 64 * kLDL * 4;      // fp32 [32][36]
    static constexpr uint32_t kXw = kX + 32 * 36 * 4;       // fp32 4 x [16][9]
    static constexpr uint32_t kGP = kXw + 4 * 16 * 9 * 4;   // fp32 [16][128] group products / prefix
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

__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity,
                                              volatile int *abort_flag, int32_t *status) {
    // Waiting threads stay suspended in try_wait (no issue slots taken from
    // the warps doing work) and wake when the phase completes; a wait that
    // outlasts 2 s of wall time gives up and flags the whole CTA.
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t start = globaltimer_ns();
    for (;;) {
        if (mbar_try_wait_sleep(bar, parity, 20000u)) return true;
        if (*abort_flag) return false;
        if (globaltimer_ns() - start > 2000000000ull) break;
    }
    *abort_flag = 1;
    set_status(status, KDA_ERR_TIMEOUT);
    return false;
}

// 16-byte shared store / load helpers
__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                       uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
                 "r"(d)
                 : "memory");
}
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}

template <int VS>
__device__ __forceinline__ uint32_t vs_off(uint32_t row, uint32_t chunk) {
    return VS == 32 ? sw64_off(row, chunk) : sw128_off(row, chunk);
}

// B-operand descriptor of a VS-wide MN-major tile (rows = K) at K step 0;
// step ks adds vs_step(ks) (start address field, in 16-byte units).
template <int VS>
__device__ __forceinline__ uint64_t vs_desc(uint32_t base, uint32_t rows) {
    return VS == 32 ? smem_desc(base, rows * 64, 512, kSw64)
                    : smem_desc(base, rows * 128, 1024, kSw128);
}
template <int VS>
__device__ __forceinline__ uint64_t vs_step(int ks) {
    return (uint64_t)(VS == 32 ? ks * 1024 : ks * 2048) >> 4;
}
// K-major 128B-swizzled operand with two 64-wide K atoms `atom` bytes apart
__device__ __forceinline__ uint64_t kmaj_step(int ks, uint32_t atom) {
    return (uint64_t)((ks >> 2) * atom + (ks & 3) * 32) >> 4;
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi) { return pack_bf16(lo, hi); }

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
    float *sX = reinterpret_cast<float *>(sm + Ly::kX);
    float *sXw = reinterpret_cast<float *>(sm + Ly::kXw);
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
        *abort_flag = 0;
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
        const int cg = t & 15, rg = t >> 4;
        const int a = cg >> 3, ch = cg & 7;
        constexpr float kLog2e = 1.4426950408889634f;
        for (int n = 0; n < nchunks; ++n) {
            const int s = n & 1;
            const int c0 = t0 + n * kChunk;
            const int L = min(kChunk, t1 - c0);
            if (!wait_or_abort(&bars[bRawFull + s], (n >> 1) & 1, abort_flag, p.status)) break;
            if (t == 0) KDA_TRACE_EVENT(n, 1);
            const uint32_t kq = sbase + Ly::kKQ + s * 32768 + a * 16384;
            const uint32_t ki = sbase + Ly::kKI + s * 16384 + a * 8192;
            // pass 0: alpha = 2^(la log2 e); in-group prefix and suffix products
            float pre[4][8], suf[4][8];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int r = rg * 4 + i;
                uint4 raw = lds128(ki + sw128_off(r, ch));
                if (r >= L) raw = make_uint4(0, 0, 0, 0);  // past the end: alpha = 1
                const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float la = (e & 1) ? bf16hi(w4[e >> 1]) : bf16lo(w4[e >> 1]);
                    pre[i][e] = ex2_approx(la * kLog2e);   // alpha for now
                }
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                float sx = 1.f;
#pragma unroll
                for (int i = 3; i >= 0; --i) {
                    suf[i][e] = sx;          // prod_{j > i} alpha_j (within the group)
                    sx *= pre[i][e];
                }
                float px = 1.f;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    px *= pre[i][e];
                    pre[i][e] = px;          // prod_{j <= i} alpha_j
                }
            }
            {
                float *gpp = sGP + rg * 128 + cg * 8;
                *reinterpret_cast<float4 *>(gpp) = make_float4(pre[3][0], pre[3][1], pre[3][2], pre[3][3]);
                *reinterpret_cast<float4 *>(gpp + 4) = make_float4(pre[3][4], pre[3][5], pre[3][6], pre[3][7]);
            }
            if (t == 0) KDA_TRACE_EVENT(n, 29);
            named_bar(kBarPrep, kPrepThreads);
            // scan over the 16 row groups, one thread per channel:
            // sGP <- exclusive prefix, sSUF <- exclusive suffix, sGL <- total
            if (t < 128) {
                float gv[16];
#pragma unroll
                for (int g = 0; g < 16; ++g) gv[g] = sGP[g * 128 + t];
                float px = 1.f;
#pragma unroll
                for (int g = 0; g < 16; ++g) {
                    sGP[g * 128 + t] = px;
                    px *= gv[g];
                }
                sGL[s * 128 + t] = px;
                float sx = rcp_approx(px);   // 1/Gam_L, once per channel
#pragma unroll
                for (int g = 15; g >= 0; --g) {
                    sSUF[g * 128 + t] = sx;
                    sx *= gv[g];
                }
            } else if (t < 128 + kChunk) {
                const int r = t - 128;
                sB[s * 64 + r] = r < L ? __bfloat162float(p.beta[(size_t)(c0 + r) * p.H + h]) : 0.f;
            }
            named_bar(kBarPrep, kPrepThreads);
            // pass 1: Gam_r = pre_group * pre[i]; 1/Gam_r = (1/Gam_L) suf_group suf[i]
            float ef[8], ci[8];
            {
                const float4 *pp = reinterpret_cast<const float4 *>(sGP + rg * 128 + cg * 8);
                const float4 *sp = reinterpret_cast<const float4 *>(sSUF + rg * 128 + cg * 8);
                const float4 p0 = pp[0], p1 = pp[1], q0 = sp[0], q1 = sp[1];
                ef[0] = p0.x; ef[1] = p0.y; ef[2] = p0.z; ef[3] = p0.w;
                ef[4] = p1.x; ef[5] = p1.y; ef[6] = p1.z; ef[7] = p1.w;
                ci[0] = q0.x; ci[1] = q0.y; ci[2] = q0.z; ci[3] = q0.w;
                ci[4] = q1.x; ci[5] = q1.y; ci[6] = q1.z; ci[7] = q1.w;
            }
            // the next chunk's pass 0 overwrites sGP: everyone must have read it
            named_bar(kBarPrep, kPrepThreads);
            if (t == 0) KDA_TRACE_EVENT(n, 30);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int r = rg * 4 + i;
                uint32_t gb[4], gib[4];
#pragma unroll
                for (int e2 = 0; e2 < 4; ++e2) {
                    gb[e2] = pack_bf16_alu(ef[2 * e2] * pre[i][2 * e2], ef[2 * e2 + 1] * pre[i][2 * e2 + 1]);
                    gib[e2] = pack_bf16_alu(ci[2 * e2] * suf[i][2 * e2], ci[2 * e2 + 1] * suf[i][2 * e2 + 1]);
                }
                if (r >= L) {  // rows past the end of the sequence are zero
#pragma unroll
                    for (int e2 = 0; e2 < 4; ++e2) gb[e2] = gib[e2] = 0u;
                }
                const uint32_t ka = kq + sw128_off(r, ch), qa = ka + 8192;
                const uint4 kr = lds128(ka), qr = lds128(qa);
                sts128(ki + sw128_off(r, ch), mul_bf16x2(kr.x, gib[0]), mul_bf16x2(kr.y, gib[1]),
                       mul_bf16x2(kr.z, gib[2]), mul_bf16x2(kr.w, gib[3]));
                sts128(ka, mul_bf16x2(kr.x, gb[0]), mul_bf16x2(kr.y, gb[1]), mul_bf16x2(kr.z, gb[2]),
                       mul_bf16x2(kr.w, gb[3]));
                sts128(qa, mul_bf16x2(qr.x, gb[0]), mul_bf16x2(qr.y, gb[1]), mul_bf16x2(qr.z, gb[2]),
                       mul_bf16x2(qr.w, gb[3]));
            }
            fence_proxy_async();
            __syncwarp();
            if (t == 0) KDA_TRACE_EVENT(n, 2);
            if (lane == 0) mbar_arrive(&bars[bKqFull + s]);
        }
    } else if (warp >= kSolve0 && warp < kSolve0 + 4) {
        // ---------------------------------------------------------- solve
        const int sw = warp - kSolve0;        // 0..3, TMEM lanes 32*sw..
        const int t = tid - kSolve0 * 32;     // 0..127
        const int g = lane >> 2, tq = lane & 3;
        for (int n = 0; n < nchunks; ++n) {
            const int s = n & 1;
            if (!wait_or_abort(&bars[bApFull], n & 1, abort_flag, p.status)) break;
            tc_fence_after();
            if (t == 0) KDA_TRACE_EVENT(n, 4);
            const uint32_t tp = sbase + Ly::kTP + s * 24576;
            {
                const int r = 32 * (sw & 1) + lane;  // row within A (sw<2) or P (sw>=2)
                uint32_t v0[32], v1[32];
                tmem_ld32(tmem_addr(tmem, 32 * sw, Ly::kTmAP), v0);
                tmem_ld32(tmem_addr(tmem, 32 * sw, Ly::kTmAP + 32), v1);
                tmem_wait_ld();
                if (t == 0) KDA_TRACE_EVENT(n, 24);
                if (sw < 2) {
                    // L = strict_lower(diag(b) A)
                    const float br = sB[s * 64 + r];
                    float *Lr = sL + r * kLDL;
#pragma unroll
                    for (int c = 0; c < 64; c += 4) {
                        const uint32_t *src = c < 32 ? &v0[c] : &v1[c - 32];
                        float4 w;
                        w.x = (c + 0 < r) ? br * __uint_as_float(src[0]) : 0.f;
                        w.y = (c + 1 < r) ? br * __uint_as_float(src[1]) : 0.f;
                        w.z = (c + 2 < r) ? br * __uint_as_float(src[2]) : 0.f;
                        w.w = (c + 3 < r) ? br * __uint_as_float(src[3]) : 0.f;
                        *reinterpret_cast<float4 *>(Lr + c) = w;
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        uint32_t o[4];
#pragma unroll
                        for (int e2 = 0; e2 < 4; ++e2) {
                            const int c = 8 * j + 2 * e2;
                            const uint32_t *src = c < 32 ? &v0[c] : &v1[c - 32];
                            const float x0 = (c <= r) ? __uint_as_float(src[0]) : 0.f;
                            const float x1 = (c + 1 <= r) ? __uint_as_float(src[1]) : 0.f;
                            o[e2] = pack2(x0, x1);
                        }
                        sts128(tp + 16384 + sw128_off(r, j), o[0], o[1], o[2], o[3]);
                    }
                }
            }
            if (t == 0) KDA_TRACE_EVENT(n, 25);
            tc_fence_before();
            named_bar(kBarSolve, 128);
            if (t == 0) mbar_arrive(&bars[bApFree]);
            if (t == 0) KDA_TRACE_EVENT(n, 5);

            // phase 1: invert the four 16x16 diagonal blocks, one block per
            // warp, one column per lane (lanes 0-15)
            if (lane < 16) {
                const int o = 16 * sw, j = lane;
                float col[16];
#pragma unroll
                for (int aa = 0; aa < 16; ++aa) col[aa] = 0.f;
#pragma unroll
                for (int aa = 0; aa < 16; ++aa) {
                    float acc = 0.f;
#pragma unroll
                    for (int m4 = 0; m4 < aa; m4 += 4) {
                        const float4 l = *reinterpret_cast<const float4 *>(sL + (o + aa) * kLDL + o + m4);
                        acc = fmaf(l.x, col[m4], acc);
                        if (m4 + 1 < aa) acc = fmaf(l.y, col[m4 + 1], acc);
                        if (m4 + 2 < aa) acc = fmaf(l.z, col[m4 + 2], acc);
                        if (m4 + 3 < aa) acc = fmaf(l.w, col[m4 + 3], acc);
                    }
                    col[aa] = (aa == j) ? 1.f : -acc;
                }
#pragma unroll
                for (int aa = 0; aa < 16; ++aa) sT[(o + aa) * kLDL + o + j] = col[aa];
                if (t == 0) KDA_TRACE_EVENT(n, 26);
            }
            named_bar(kBarSolve, 128);
            if (t == 0) KDA_TRACE_EVENT(n, 6);

            // phase 2: 32x32 blocks: T21 = -T22 (L21 T11), one 16x8 tile per warp
            {
                const int pb = sw >> 1, nt = sw & 1;
                const int R1 = 32 * pb + 16, C0 = 32 * pb;
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int kk = 0; kk < 16; kk += 8) {
                    const uint32_t af[4] = {
                        tf32_bits(sL[(R1 + g) * kLDL + C0 + kk + tq]),
                        tf32_bits(sL[(R1 + g + 8) * kLDL + C0 + kk + tq]),
                        tf32_bits(sL[(R1 + g) * kLDL + C0 + kk + tq + 4]),
                        tf32_bits(sL[(R1 + g + 8) * kLDL + C0 + kk + tq + 4])};
                    const uint32_t bfr[2] = {tf32_bits(sT[(C0 + kk + tq) * kLDL + C0 + 8 * nt + g]),
                                             tf32_bits(sT[(C0 + kk + tq + 4) * kLDL + C0 + 8 * nt + g])};
                    mma_tf32_16x8x8(acc, af, bfr);
                }
                float *xw = sXw + sw * 16 * 9;
                xw[g * 9 + 2 * tq] = acc[0];
                xw[g * 9 + 2 * tq + 1] = acc[1];
                xw[(g + 8) * 9 + 2 * tq] = acc[2];
                xw[(g + 8) * 9 + 2 * tq + 1] = acc[3];
                __syncwarp();
                float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int kk = 0; kk < 16; kk += 8) {
                    const uint32_t af[4] = {
                        tf32_bits(sT[(R1 + g) * kLDL + R1 + kk + tq]),
                        tf32_bits(sT[(R1 + g + 8) * kLDL + R1 + kk + tq]),
                        tf32_bits(sT[(R1 + g) * kLDL + R1 + kk + tq + 4]),
                        tf32_bits(sT[(R1 + g + 8) * kLDL + R1 + kk + tq + 4])};
                    const uint32_t bfr[2] = {tf32_bits(xw[(kk + tq) * 9 + g]),
                                             tf32_bits(xw[(kk + tq + 4) * 9 + g])};
                    mma_tf32_16x8x8(d, af, bfr);
                }
                float *o = sT + R1 * kLDL + C0 + 8 * nt;
                o[g * kLDL + 2 * tq] = -d[0];
                o[g * kLDL + 2 * tq + 1] = -d[1];
                o[(g + 8) * kLDL + 2 * tq] = -d[2];
                o[(g + 8) * kLDL + 2 * tq + 1] = -d[3];
            }
            named_bar(kBarSolve, 128);
            if (t == 0) KDA_TRACE_EVENT(n, 7);

            // phase 3: 64x64: T_BA = -T_B (L_BA T_A); warp = (m tile, pair of n
            // tiles).  Blocks above the diagonal blocks of T are zero.
            {
                const int mt = sw & 1, nb = 2 * (sw >> 1);
                const int rr = 32 + 16 * mt;
                float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
                for (int kk = 0; kk < 32; kk += 8) {
                    const uint32_t af[4] = {tf32_bits(sL[(rr + g) * kLDL + kk + tq]),
                                            tf32_bits(sL[(rr + g + 8) * kLDL + kk + tq]),
                                            tf32_bits(sL[(rr + g) * kLDL + kk + tq + 4]),
                                            tf32_bits(sL[(rr + g + 8) * kLDL + kk + tq + 4])};
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const int c = 8 * (nb + q) + g;
                        const uint32_t bfr[2] = {tf32_bits(sT[(kk + tq) * kLDL + c]),
                                                 tf32_bits(sT[(kk + tq + 4) * kLDL + c])};
                        mma_tf32_16x8x8(acc[q], af, bfr);
                    }
                }
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    float *o = sX + (16 * mt) * 36 + 8 * (nb + q);
                    o[g * 36 + 2 * tq] = acc[q][0];
                    o[g * 36 + 2 * tq + 1] = acc[q][1];
                    o[(g + 8) * 36 + 2 * tq] = acc[q][2];
                    o[(g + 8) * 36 + 2 * tq + 1] = acc[q][3];
                }
                if (t == 0) KDA_TRACE_EVENT(n, 27);
                named_bar(kBarSolve, 128);
                float d[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
                for (int kk = 0; kk < 32; kk += 8) {
                    const uint32_t af[4] = {tf32_bits(sT[(rr + g) * kLDL + 32 + kk + tq]),
                                            tf32_bits(sT[(rr + g + 8) * kLDL + 32 + kk + tq]),
                                            tf32_bits(sT[(rr + g) * kLDL + 32 + kk + tq + 4]),
                                            tf32_bits(sT[(rr + g + 8) * kLDL + 32 + kk + tq + 4])};
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const int cc = 8 * (nb + q);
                        const uint32_t bfr[2] = {tf32_bits(sX[(kk + tq) * 36 + cc + g]),
                                                 tf32_bits(sX[(kk + tq + 4) * 36 + cc + g])};
                        mma_tf32_16x8x8(d[q], af, bfr);
                    }
                }
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    float *o = sT + rr * kLDL + 8 * (nb + q);
                    o[g * kLDL + 2 * tq] = -d[q][0];
                    o[g * kLDL + 2 * tq + 1] = -d[q][1];
                    o[(g + 8) * kLDL + 2 * tq] = -d[q][2];
                    o[(g + 8) * kLDL + 2 * tq + 1] = -d[q][3];
                }
            }
            named_bar(kBarSolve, 128);
            if (t == 0) KDA_TRACE_EVENT(n, 8);

            // Tb = T diag(b) -> bf16, rows 0..63 of the Tb|0|P tile
            {
                const int r = t >> 1, half = t & 1;
                const float *Tr = sT + r * kLDL + 32 * half;
                const float *bs = sB + s * 64 + 32 * half;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float4 t0v = *reinterpret_cast<const float4 *>(Tr + 8 * j);
                    const float4 t1v = *reinterpret_cast<const float4 *>(Tr + 8 * j + 4);
                    const float4 b0v = *reinterpret_cast<const float4 *>(bs + 8 * j);
                    const float4 b1v = *reinterpret_cast<const float4 *>(bs + 8 * j + 4);
                    sts128(tp + sw128_off(r, 4 * half + j), pack2(t0v.x * b0v.x, t0v.y * b0v.y),
                           pack2(t0v.z * b0v.z, t0v.w * b0v.w), pack2(t1v.x * b1v.x, t1v.y * b1v.y),
                           pack2(t1v.z * b1v.z, t1v.w * b1v.w));
                }
            }
            if (t == 0) KDA_TRACE_EVENT(n, 28);
            fence_proxy_async();
            named_bar(kBarSolve, 128);
            if (t == 0) mbar_arrive(&bars[bTbFull + s]);
            if (t == 0) KDA_TRACE_EVENT(n, 9);

            // W = Tb Kg (TMEM, fp32) -> -W as bf16 over the Kg rows of this stage
            if (sw < 2) {
                if (!wait_or_abort(&bars[bWaccFull], n & 1, abort_flag, p.status)) break;
                tc_fence_after();
                if (t == 0) KDA_TRACE_EVENT(n, 11);
                const int r = 32 * sw + lane;
                const uint32_t kq = sbase + Ly::kKQ + s * 32768;
#pragma unroll
                for (int blk = 0; blk < 4; ++blk) {
                    uint32_t v[32];
                    tmem_ld32(tmem_addr(tmem, 32 * sw, Ly::kTmW + 32 * blk), v);
                    tmem_wait_ld();
                    const int aa = blk >> 1;
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        uint32_t o[4];
#pragma unroll
                        for (int e2 = 0; e2 < 4; ++e2) {
                            const int c = 8 * j + 2 * e2;
                            o[e2] = pack2(-__uint_as_float(v[c]), -__uint_as_float(v[c + 1]));
                        }
                        const int chunk = 4 * (blk & 1) + j;
                        sts128(kq + aa * 16384 + sw128_off(r, chunk), o[0], o[1], o[2], o[3]);
                    }
                }
                fence_proxy_async();
                tc_fence_before();
                __syncwarp();
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
    if (warp == kMmaK) {
        tc_fence_after();
        tmem_dealloc(tmem, Ly::kTmCols);
    }
}

// ---------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

// [T, H, D] bf16 tensor; box = {bx channels, 1 head, 64 tokens}
bool make_map(CUtensorMap *m, const void *base, int T, int H, int D, int bx,
              CUtensorMapSwizzle swz) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T};
    const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
    const cuuint32_t box[3] = {(cuuint32_t)bx, 1, (cuuint32_t)kChunk};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int VS>
cudaError_t launch_vs(const ForwardArgs &a, cudaStream_t s) {
    CUtensorMap mq, mk, mla, mv;
    const int T = a.T > 0 ? a.T : 1;
    if (!make_map(&mq, a.q, T, a.H, kDK, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mk, a.k, T, a.H, kDK, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mla, a.log_alpha, T, a.H, kDK, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mv, a.v, T, a.H, kDV, VS,
                  VS == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B))
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
    return a.io_dtype == KDA_BF16 && a.gate_dtype == KDA_BF16 && a.Dk == kDK && a.Dv == kDV;
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
