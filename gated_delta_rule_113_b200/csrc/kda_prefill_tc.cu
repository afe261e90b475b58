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
// One CTA owns one (sequence, head, VS-wide slice of d_v): everything after
// MMA_W is separable over value columns.  Warp roles (15 warps):
//   0-3   chain: thread c owns state row c (fp32 registers); warps 0-1 turn
//         U into the bf16 operand, warps 2-3 write the outputs
//   4-7   prep: gates and the scaled operands, in place over the TMA tiles
//   8-11  solve: triangular inverse, P mask, W -> bf16 operand
//   12    TMA producer
//   13    key-side MMA issuer (MMA_AP, MMA_W, MMA_0); owns TMEM
//   14    chain MMA issuer (MMA_1, MMA_2, MMA_3)
// Two pipeline stages of operand tiles let the key-side work of chunk n+1
// overlap the sequential state chain of chunk n.  All waits are bounded.
#include <cuda.h>

#include "kda_internal.cuh"
#include "sm100.cuh"

namespace kda {
namespace {

using namespace sm100;

constexpr int kWarps = 15;
constexpr int kThreads = kWarps * 32;
constexpr int kDK = 128;           // key width handled by this kernel
constexpr int kDV = 128;           // value width handled by this kernel
constexpr int kLDL = 68;           // fp32 row stride of the solve scratch

enum Role { kChain0 = 0, kPrep0 = 4, kSolve0 = 8, kTma = 12, kMmaK = 13, kMmaC = 14 };
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
    static constexpr uint32_t kGP = kXw + 4 * 16 * 9 * 4;   // fp32 [8][128]
    static constexpr uint32_t kGL = kGP + 8 * 128 * 4;      // fp32 [2][128]
    static constexpr uint32_t kB = kGL + 2 * 128 * 4;       // fp32 [2][64]
    static constexpr uint32_t kBar = kB + 2 * 64 * 4;       // mbarriers
    static constexpr uint32_t kNumBars = 32;
    static constexpr uint32_t kMisc = kBar + kNumBars * 8;  // tmem base, abort flag
    static constexpr uint32_t kSize = kMisc + 16;
    static constexpr uint32_t kAlloc = kSize + 1024;        // + alignment slack
    static_assert(kAlloc <= 232448, "shared memory budget exceeded");
    static_assert(VS == 32 || VS == 64, "value slice must be 32 or 64");

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
    bDrainK = 23,    // issuer drains before exit
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
    for (uint32_t i = 0; i < (1u << 22); ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (i > 64) __nanosleep(64);
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

// B-operand descriptor of a VS-wide MN-major tile (rows = K), K step ks of 16 rows.
template <int VS>
__device__ __forceinline__ uint64_t vs_desc(uint32_t base, int ks, uint32_t rows) {
    return VS == 32 ? smem_desc(base + ks * 1024, rows * 64, 512, kSw64)
                    : smem_desc(base + ks * 2048, rows * 128, 1024, kSw128);
}

template <int VS>
__global__ void __launch_bounds__(kThreads, 1)
prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_la,
                  const __grid_constant__ CUtensorMap tm_v, TcParams p) {
    using Ly = Layout<VS>;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + Ly::kBar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + Ly::kMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + Ly::kMisc + 4);
    float *sL = reinterpret_cast<float *>(sm + Ly::kL);
    float *sT = reinterpret_cast<float *>(sm + Ly::kT);
    float *sX = reinterpret_cast<float *>(sm + Ly::kX);
    float *sXw = reinterpret_cast<float *>(sm + Ly::kXw);
    float *sGP = reinterpret_cast<float *>(sm + Ly::kGP);
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
            if (i == bKqFull || i == bKqFull + 1) cnt = 4;
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
    // zero rows 64..127 of both Tb|0|P tiles (never written afterwards)
    for (int i = tid; i < 2 * 512; i += kThreads) {
        const int s = i / 512, j = i % 512;
        sts128(sbase + Ly::kTP + s * 24576 + 8192 + j * 16, 0, 0, 0, 0);
    }
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
    } else if (warp >= kPrep0 && warp < kPrep0 + 4) {
        // ----------------------------------------------------------- prep
        const int t = tid - kPrep0 * 32;
        const int cg = t & 15, rg = t >> 4;
        const int a = cg >> 3, ch = cg & 7;
        constexpr float kLog2e = 1.4426950408889634f;
        for (int n = 0; n < nchunks; ++n) {
            const int s = n & 1;
            const int c0 = t0 + n * kChunk;
            const int L = min(kChunk, t1 - c0);
            if (!wait_or_abort(&bars[bRawFull + s], (n >> 1) & 1, abort_flag, p.status)) break;
            const uint32_t kq = sbase + Ly::kKQ + s * 32768 + a * 16384;
            const uint32_t ki = sbase + Ly::kKI + s * 16384 + a * 8192;
            float alpha[8][8];
            float gp[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) gp[e] = 1.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int r = rg * 8 + i;
                const uint4 raw = lds128(ki + sw128_off(r, ch));
                const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float la = (e & 1) ? bf16hi(w4[e >> 1]) : bf16lo(w4[e >> 1]);
                    const float al = r < L ? exp2f(la * kLog2e) : 1.f;
                    alpha[i][e] = al;
                    gp[e] *= al;
                }
            }
            float *gpp = sGP + rg * 128 + cg * 8;
#pragma unroll
            for (int e = 0; e < 8; ++e) gpp[e] = gp[e];
            named_bar(kBarPrep, 128);
            float ef[8], er[8], igl[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) { ef[e] = 1.f; er[e] = 1.f; }
            for (int g = 0; g < 8; ++g) {
                const float *row = sGP + g * 128 + cg * 8;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    if (g < rg) ef[e] *= row[e];
                    if (g > rg) er[e] *= row[e];
                }
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float glv = ef[e] * gp[e] * er[e];
                igl[e] = 1.f / glv;
                if (rg == 0) sGL[s * 128 + cg * 8 + e] = glv;
            }
            // Ki = K / Gam, walking rows backwards: 1/Gam_r = (1/Gam_L) prod_{j>r} alpha_j
            float sfx[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) sfx[e] = er[e];
#pragma unroll
            for (int i = 7; i >= 0; --i) {
                const int r = rg * 8 + i;
                const uint4 kr = lds128(kq + sw128_off(r, ch));
                const uint32_t kw[4] = {kr.x, kr.y, kr.z, kr.w};
                uint32_t o[4];
#pragma unroll
                for (int e2 = 0; e2 < 4; ++e2) {
                    float k0 = bf16lo(kw[e2]), k1 = bf16hi(kw[e2]);
                    if (r >= L) { k0 = 0.f; k1 = 0.f; }
                    o[e2] = pack_bf16(k0 * igl[2 * e2] * sfx[2 * e2],
                                      k1 * igl[2 * e2 + 1] * sfx[2 * e2 + 1]);
                }
                sts128(ki + sw128_off(r, ch), o[0], o[1], o[2], o[3]);
#pragma unroll
                for (int e = 0; e < 8; ++e) sfx[e] *= alpha[i][e];
            }
            // Qg = Q * Gam, Kg = K * Gam in place, walking rows forwards
            float pf[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) pf[e] = ef[e];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int r = rg * 8 + i;
#pragma unroll
                for (int e = 0; e < 8; ++e) pf[e] *= alpha[i][e];
                const uint32_t ka = kq + sw128_off(r, ch), qa = ka + 8192;
                const uint4 kr = lds128(ka), qr = lds128(qa);
                const uint32_t kw[4] = {kr.x, kr.y, kr.z, kr.w};
                const uint32_t qw[4] = {qr.x, qr.y, qr.z, qr.w};
                uint32_t ok[4], oq[4];
#pragma unroll
                for (int e2 = 0; e2 < 4; ++e2) {
                    float k0 = bf16lo(kw[e2]), k1 = bf16hi(kw[e2]);
                    float q0 = bf16lo(qw[e2]), q1 = bf16hi(qw[e2]);
                    if (r >= L) { k0 = k1 = q0 = q1 = 0.f; }
                    ok[e2] = pack_bf16(k0 * pf[2 * e2], k1 * pf[2 * e2 + 1]);
                    oq[e2] = pack_bf16(q0 * pf[2 * e2], q1 * pf[2 * e2 + 1]);
                }
                sts128(ka, ok[0], ok[1], ok[2], ok[3]);
                sts128(qa, oq[0], oq[1], oq[2], oq[3]);
            }
            if (t < kChunk)
                sB[s * 64 + t] = t < L ? __bfloat162float(p.beta[(size_t)(c0 + t) * p.H + h]) : 0.f;
            fence_proxy_async();
            named_bar(kBarPrep, 128);   // sGP reuse + beta visible before release
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
            const uint32_t tp = sbase + Ly::kTP + s * 24576;
            {
                const int r = 32 * (sw & 1) + lane;  // row within A (sw<2) or P (sw>=2)
                uint32_t v0[32], v1[32];
                tmem_ld32(tmem_addr(tmem, 32 * sw, Ly::kTmAP), v0);
                tmem_ld32(tmem_addr(tmem, 32 * sw, Ly::kTmAP + 32), v1);
                tmem_wait_ld();
                if (sw < 2) {
                    const float br = sB[s * 64 + r];
                    float *Lr = sL + r * kLDL;
#pragma unroll
                    for (int c = 0; c < 64; c += 4) {
                        float4 w;
                        const uint32_t *src = c < 32 ? &v0[c] : &v1[c - 32];
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
                            o[e2] = pack_bf16(x0, x1);
                        }
                        sts128(tp + 16384 + sw128_off(r, j), o[0], o[1], o[2], o[3]);
                    }
                }
            }
            tc_fence_before();
            named_bar(kBarSolve, 128);
            if (t == 0) mbar_arrive(&bars[bApFree]);

            // phase 1: invert the four 16x16 diagonal blocks (column per thread)
            if (t < 64) {
                const int blk = t >> 4, j = t & 15, o = 16 * blk;
                float col[16];
#pragma unroll
                for (int aa = 0; aa < 16; ++aa) {
                    float acc = 0.f;
#pragma unroll
                    for (int m = 0; m < aa; ++m) acc = fmaf(sL[(o + aa) * kLDL + o + m], col[m], acc);
                    col[aa] = (aa == j) ? 1.f : -acc;
                }
#pragma unroll
                for (int aa = 0; aa < 16; ++aa) sT[(o + aa) * kLDL + o + j] = col[aa];
            }
            named_bar(kBarSolve, 128);

            // phase 2: 32x32 blocks: T21 = -T22 (L21 T11), one 16x8 tile per warp
            {
                const int pb = sw >> 1, nt = sw & 1;
                const int R1 = 32 * pb + 16, C0 = 32 * pb;
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int kk = 0; kk < 16; kk += 8) {
                    const uint32_t af[4] = {
                        to_tf32(sL[(R1 + g) * kLDL + C0 + kk + tq]),
                        to_tf32(sL[(R1 + g + 8) * kLDL + C0 + kk + tq]),
                        to_tf32(sL[(R1 + g) * kLDL + C0 + kk + tq + 4]),
                        to_tf32(sL[(R1 + g + 8) * kLDL + C0 + kk + tq + 4])};
                    const uint32_t bfr[2] = {to_tf32(sT[(C0 + kk + tq) * kLDL + C0 + 8 * nt + g]),
                                             to_tf32(sT[(C0 + kk + tq + 4) * kLDL + C0 + 8 * nt + g])};
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
                        to_tf32(sT[(R1 + g) * kLDL + R1 + kk + tq]),
                        to_tf32(sT[(R1 + g + 8) * kLDL + R1 + kk + tq]),
                        to_tf32(sT[(R1 + g) * kLDL + R1 + kk + tq + 4]),
                        to_tf32(sT[(R1 + g + 8) * kLDL + R1 + kk + tq + 4])};
                    const uint32_t bfr[2] = {to_tf32(xw[(kk + tq) * 9 + g]),
                                             to_tf32(xw[(kk + tq + 4) * 9 + g])};
                    mma_tf32_16x8x8(d, af, bfr);
                }
                float *o = sT + R1 * kLDL + C0 + 8 * nt;
                o[g * kLDL + 2 * tq] = -d[0];
                o[g * kLDL + 2 * tq + 1] = -d[1];
                o[(g + 8) * kLDL + 2 * tq] = -d[2];
                o[(g + 8) * kLDL + 2 * tq + 1] = -d[3];
            }
            named_bar(kBarSolve, 128);

            // phase 3: 64x64: T_BA = -T_B (L_BA T_A); warp = (m tile, pair of n tiles)
            {
                const int mt = sw & 1, nb = 2 * (sw >> 1);
                float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
                for (int kk = 0; kk < 32; kk += 8) {
                    const int rr = 32 + 16 * mt;
                    const uint32_t af[4] = {to_tf32(sL[(rr + g) * kLDL + kk + tq]),
                                            to_tf32(sL[(rr + g + 8) * kLDL + kk + tq]),
                                            to_tf32(sL[(rr + g) * kLDL + kk + tq + 4]),
                                            to_tf32(sL[(rr + g + 8) * kLDL + kk + tq + 4])};
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const int cc = 8 * (nb + q);
                        // T_A is lower triangular: entries above the diagonal are zero
                        const int k0 = kk + tq, k1 = kk + tq + 4, c = cc + g;
                        const uint32_t bfr[2] = {to_tf32(c <= k0 ? sT[k0 * kLDL + c] : 0.f),
                                                 to_tf32(c <= k1 ? sT[k1 * kLDL + c] : 0.f)};
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
                named_bar(kBarSolve, 128);
                float d[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
                for (int kk = 0; kk < 32; kk += 8) {
                    const int rr = 32 + 16 * mt;
                    // T_B lower triangular (rows rr+g.., cols 32+k)
                    const int r0 = 16 * mt + g, r1 = r0 + 8;
                    const int k0 = kk + tq, k1 = kk + tq + 4;
                    const uint32_t af[4] = {
                        to_tf32(k0 <= r0 ? sT[(rr + g) * kLDL + 32 + k0] : 0.f),
                        to_tf32(k0 <= r1 ? sT[(rr + g + 8) * kLDL + 32 + k0] : 0.f),
                        to_tf32(k1 <= r0 ? sT[(rr + g) * kLDL + 32 + k1] : 0.f),
                        to_tf32(k1 <= r1 ? sT[(rr + g + 8) * kLDL + 32 + k1] : 0.f)};
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const int cc = 8 * (nb + q);
                        const uint32_t bfr[2] = {to_tf32(sX[k0 * 36 + cc + g]),
                                                 to_tf32(sX[k1 * 36 + cc + g])};
                        mma_tf32_16x8x8(d[q], af, bfr);
                    }
                }
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    float *o = sT + (32 + 16 * mt) * kLDL + 8 * (nb + q);
                    o[g * kLDL + 2 * tq] = -d[q][0];
                    o[g * kLDL + 2 * tq + 1] = -d[q][1];
                    o[(g + 8) * kLDL + 2 * tq] = -d[q][2];
                    o[(g + 8) * kLDL + 2 * tq + 1] = -d[q][3];
                }
            }
            named_bar(kBarSolve, 128);

            // Tb = T diag(b) -> bf16, rows 0..63 of the Tb|0|P tile
            {
                const int r = t >> 1, half = t & 1;
                const float *Tr = sT + r * kLDL;
                const float *bs = sB + s * 64;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    uint32_t o[4];
#pragma unroll
                    for (int e2 = 0; e2 < 4; ++e2) {
                        const int c = 32 * half + 8 * j + 2 * e2;
                        const float x0 = c <= r ? Tr[c] * bs[c] : 0.f;
                        const float x1 = c + 1 <= r ? Tr[c + 1] * bs[c + 1] : 0.f;
                        o[e2] = pack_bf16(x0, x1);
                    }
                    sts128(tp + sw128_off(r, 4 * half + j), o[0], o[1], o[2], o[3]);
                }
            }
            fence_proxy_async();
            named_bar(kBarSolve, 128);
            if (t == 0) mbar_arrive(&bars[bTbFull + s]);

            // W = Tb Kg (TMEM, fp32) -> -W as bf16 over the Kg rows of this stage
            if (sw < 2) {
                if (!wait_or_abort(&bars[bWaccFull], n & 1, abort_flag, p.status)) break;
                tc_fence_after();
                const int r = 32 * sw + lane;
                const uint32_t kq = sbase + Ly::kKQ + s * 32768;
#pragma unroll
                for (int blk = 0; blk < 4; ++blk) {
                    uint32_t v[32];
                    tmem_ld32(tmem_addr(tmem, 32 * sw, Ly::kTmW + 32 * blk), v);
                    tmem_wait_ld();
                    const int a = blk >> 1;
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        uint32_t o[4];
#pragma unroll
                        for (int e2 = 0; e2 < 4; ++e2) {
                            const int c = 8 * j + 2 * e2;
                            o[e2] = pack_bf16(-__uint_as_float(v[c]), -__uint_as_float(v[c + 1]));
                        }
                        const int chunk = 4 * (blk & 1) + j;
                        sts128(kq + a * 16384 + sw128_off(r, chunk), o[0], o[1], o[2], o[3]);
                    }
                }
                fence_proxy_async();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[bWReady + s]);
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
                if (!wait_or_abort(&bars[bKqFull + s], (n >> 1) & 1, abort_flag, p.status)) break;
                if (n >= 1 && !wait_or_abort(&bars[bApFree], (n - 1) & 1, abort_flag, p.status)) break;
                tc_fence_after();
                for (int ks = 0; ks < 8; ++ks) {
                    const uint64_t ad = smem_desc(kq + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024, kSw128);
                    const uint64_t bd = smem_desc(ki + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024, kSw128);
                    mma_bf16(tmem + Ly::kTmAP, ad, bd, kIdAP, ks > 0);
                }
                mma_commit(&bars[bApFull]);

                if (!wait_or_abort(&bars[bTbFull + s], (n >> 1) & 1, abort_flag, p.status)) break;
                if (n >= 1 && !wait_or_abort(&bars[bWReady + ((n - 1) & 1)], ((n - 1) >> 1) & 1,
                                             abort_flag, p.status))
                    break;
                tc_fence_after();
                for (int ks = 0; ks < 4; ++ks) {
                    const uint64_t ad = smem_desc(tp + ks * 32, 16, 1024, kSw128);
                    const uint64_t bd = smem_desc(kq + ks * 2048, 16384, 1024, kSw128);
                    mma_bf16(tmem + Ly::kTmW, ad, bd, kIdW, ks > 0);
                }
                mma_commit(&bars[bWaccFull]);

                if (n >= 2 && !wait_or_abort(&bars[bD1Free + s], ((n - 2) >> 1) & 1, abort_flag,
                                             p.status))
                    break;
                tc_fence_after();
                for (int ks = 0; ks < 4; ++ks) {
                    const uint64_t ad = smem_desc(tp + ks * 32, 16, 1024, kSw128);
                    mma_bf16(tmem + Ly::kTmD1 + s * VS, ad, vs_desc<VS>(vt, ks, 64), kIdV, ks > 0);
                }
                mma_commit(&bars[bU0Done + s]);
            }
            mma_commit(&bars[bDrainK]);
            mbar_wait(&bars[bDrainK], 0);
        }
    } else if (warp == kMmaC) {
        // ------------------------------------------------- chain MMA issuer
        if (lane == 0) {
            constexpr uint32_t kIdV = idesc_bf16(128, VS, 0, 1);
            constexpr uint32_t kIdS = idesc_bf16(128, VS, 1, 1);
            const uint32_t sb = sbase + Ly::kSB, ub = sbase + Ly::kUB;
            for (int n = 0; n < nchunks; ++n) {
                const int s = n & 1;
                const uint32_t kq = sbase + Ly::kKQ + s * 32768;
                const uint32_t ki = sbase + Ly::kKI + s * 16384;
                const uint32_t tp = sbase + Ly::kTP + s * 24576;
                const uint32_t d1 = tmem + Ly::kTmD1 + s * VS;
                if (!wait_or_abort(&bars[bWReady + s], (n >> 1) & 1, abort_flag, p.status)) break;
                if (!wait_or_abort(&bars[bU0Done + s], (n >> 1) & 1, abort_flag, p.status)) break;
                if (!wait_or_abort(&bars[bSbFull], n & 1, abort_flag, p.status)) break;
                tc_fence_after();
                for (int ks = 0; ks < 8; ++ks) {
                    const uint64_t ad = smem_desc(kq + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024, kSw128);
                    mma_bf16(d1, ad, vs_desc<VS>(sb, ks, 128), kIdV, 1);
                }
                mma_commit(&bars[bUFull]);
                if (!wait_or_abort(&bars[bUbFull], n & 1, abort_flag, p.status)) break;
                tc_fence_after();
                for (int ks = 0; ks < 4; ++ks) {
                    const uint64_t ad = smem_desc(ki + ks * 2048, 8192, 1024, kSw128);
                    mma_bf16(tmem + Ly::kTmD2, ad, vs_desc<VS>(ub, ks, 64), kIdS, ks > 0);
                }
                mma_commit(&bars[bDsFull]);
                for (int ks = 0; ks < 4; ++ks) {
                    const uint64_t ad = smem_desc(tp + 8192 + ks * 32, 16, 1024, kSw128);
                    mma_bf16(d1, ad, vs_desc<VS>(ub, ks, 64), kIdV, 1);
                }
                mma_commit(&bars[bOFull + s]);
                mma_commit(&bars[bStageFree + s]);
            }
            mma_commit(&bars[bDrainC]);
            mbar_wait(&bars[bDrainC], 0);
        }
    } else {
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
        float gl_cur = 1.f;
        bool ok = true;
        for (int n = 0; n <= nchunks && ok; ++n) {
            if (n > 0) {
                // S <- Diag(Gam_L) (S + dS) for chunk n-1
                if (!wait_or_abort(&bars[bDsFull], (n - 1) & 1, abort_flag, p.status)) { ok = false; break; }
                tc_fence_after();
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
                // outputs of the last chunk
                if (wq >= 2 && n > 0) {
                    const int m = n - 1, sm1 = m & 1;
                    if (!wait_or_abort(&bars[bOFull + sm1], (m >> 1) & 1, abort_flag, p.status)) { ok = false; break; }
                    tc_fence_after();
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
                                w.x = pack_bf16(__uint_as_float(v[e]), __uint_as_float(v[e + 1]));
                                w.y = pack_bf16(__uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
                                w.z = pack_bf16(__uint_as_float(v[e + 4]), __uint_as_float(v[e + 5]));
                                w.w = pack_bf16(__uint_as_float(v[e + 6]), __uint_as_float(v[e + 7]));
                                *reinterpret_cast<uint4 *>(dst + e) = w;
                            }
                        }
                    }
                }
                break;
            }
            const int s = n & 1;
            // Gam_L of this chunk (prep done) and the bf16 state operand
            if (!wait_or_abort(&bars[bKqFull + s], (n >> 1) & 1, abort_flag, p.status)) { ok = false; break; }
            gl_cur = sGL[s * 128 + c];
            {
                const uint32_t sb = sbase + Ly::kSB;
#pragma unroll
                for (int j = 0; j < VS / 8; ++j) {
                    sts128(sb + vs_off<VS>(c, j), pack_bf16(S[8 * j], S[8 * j + 1]),
                           pack_bf16(S[8 * j + 2], S[8 * j + 3]), pack_bf16(S[8 * j + 4], S[8 * j + 5]),
                           pack_bf16(S[8 * j + 6], S[8 * j + 7]));
                }
            }
            fence_proxy_async();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[bSbFull]);

            if (wq < 2) {
                // U rows: D1 lanes 0..63 -> bf16 operand
                if (!wait_or_abort(&bars[bUFull], n & 1, abort_flag, p.status)) { ok = false; break; }
                tc_fence_after();
                const uint32_t ub = sbase + Ly::kUB;
#pragma unroll
                for (int j = 0; j < VS; j += 32) {
                    uint32_t v[32];
                    tmem_ld32(tmem_addr(tmem, 32 * wq, Ly::kTmD1 + s * VS + j), v);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; e += 8) {
                        sts128(ub + vs_off<VS>(c, (j + e) / 8),
                               pack_bf16(__uint_as_float(v[e]), __uint_as_float(v[e + 1])),
                               pack_bf16(__uint_as_float(v[e + 2]), __uint_as_float(v[e + 3])),
                               pack_bf16(__uint_as_float(v[e + 4]), __uint_as_float(v[e + 5])),
                               pack_bf16(__uint_as_float(v[e + 6]), __uint_as_float(v[e + 7])));
                    }
                }
                fence_proxy_async();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[bUbFull]);
            } else if (n > 0) {
                // outputs of chunk n-1: D1 lanes 64..127
                const int m = n - 1, sm1 = m & 1;
                if (!wait_or_abort(&bars[bOFull + sm1], (m >> 1) & 1, abort_flag, p.status)) { ok = false; break; }
                tc_fence_after();
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
                            w.x = pack_bf16(__uint_as_float(v[e]), __uint_as_float(v[e + 1]));
                            w.y = pack_bf16(__uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
                            w.z = pack_bf16(__uint_as_float(v[e + 4]), __uint_as_float(v[e + 5]));
                            w.w = pack_bf16(__uint_as_float(v[e + 6]), __uint_as_float(v[e + 7]));
                            *reinterpret_cast<uint4 *>(dst + e) = w;
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[bD1Free + sm1]);
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
