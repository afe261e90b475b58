// kda_backward_tc.cu -- gradients of the KDA recurrence through the chunk
// form, on tensor cores (bf16 operands, fp32 accumulation).
//
// The page "Kimi K3: Open Frontier Intelligence and Implementation
// Framework" (section "Hybrid Attention Mechanism", KDA bullet) evaluates the
// delta rule with a channel-wise forget gate chunk by chunk with dense
// tensor-core tiles; the model built on it is trained, so the same chunk form
// is run backwards here.  Per chunk of C = 64 tokens (Gam = running decay,
// Qg = Q Gam, Kg = K Gam, Ki = K / Gam, b = beta) the forward is
//   A_full = Kg Ki^T,  A = strict_lower(diag(b) A_full),  T = (I + A)^{-1},
//   Tb = T diag(b),  W = Tb Kg,  U = Tb V - W S,  P = lower_incl(Qg Ki^T),
//   O = Qg S + P U,  S' = Diag(Gam_L) (S + Ki^T U)
// and, given dO and dX = Diag(Gam_L) dS' (the gradient reaching the
// bracket), the backward is
//   dU  = P^T dO + Ki dX                 dP  = lower_incl(dO U^T)
//   dQg = dO S^T + dP Ki                 dKi = U dX^T + dP^T Qg + dAf^T Kg
//   dW  = -dU S^T                        dTb = dU V^T + dW Kg^T
//   dV  = Tb^T dU                        dKg = Tb^T dW + dAf Ki
//   dT  = dTb diag(b)                    dA  = strict_lower(-T^T dT T^T)
//   dAf = diag(b) dA                     db  = colsum(T * dTb) + rowsum(dA * A_full)
//   dQ = dQg Gam,  dK = dKg Gam + dKi / Gam,
//   dG = dKg * Kg + dQg * Qg - dKi * Ki  (+ rowsum(X * dX) on the last row,
//        X = S + Ki^T U),  dlog_alpha = reverse cumulative sum of dG,
// and the state gradient entering the chunk is
//   dS = dX + Qe^T dO + (-W)^T (Ki dX),  Qe = Qg - P W.
//
// Three passes after the forward's two (which leave the operand packets and,
// with the state store switched on, every chunk's entering state S_j):
//   rchain_kernel   one CTA per (sequence, head, 32-wide value slice) walks
//                   the chunks backwards with the packets' tiles transposed:
//                   dX_j = Gam_L,j dS_{j+1};  dU_j = Ki_j dX_j;
//                   dS_j = dX_j + [-W; Qe]_j^T [dU_j; dO_j]  (tcgen05, TMEM)
//                   and stores dX_j of every chunk;
//   assemble_kernel one CTA per (chunk, head): the gradient algebra above
//                   with warp-level bf16 tensor-core products (mma.sync) over
//                   swizzled shared-memory tiles; every gradient row is
//                   written once, so the result is bitwise reproducible.
#include <string.h>

#include "kda_internal.cuh"
#include "kda_tc_common.cuh"
#include "sm100.cuh"

namespace kda {
namespace {

using namespace sm100;
using namespace tc;

// ============================================================ reverse chain
constexpr int kRcVs = 32;               // value columns per CTA
constexpr int kRcWarps = 6;             // 0-3 chain, 4 loader, 5 MMA
constexpr int kRcThreads = kRcWarps * 32;
constexpr int kRcStages = 3;
enum RcBars {
    rbFull = 0,      // [3] stage landed: [-W; Qe], Ki, Gam_L, dO
    rbFree = 3,      // [3] every product reading the stage done
    rbXbFull = 6,    // count 4: bf16 dX written
    rbDuAcc = 7,     // dU = Ki dX complete
    rbDuFull = 8,    // count 4: bf16 dU written into the stage
    rbDsAcc = 9,     // [2] [-W; Qe]^T [dU; dO] complete, by step parity
    rbDrain = 11,
    rbNum = 12
};
struct RcLayout {
    // stage: [-W; Qe] 32 KB | Ki 16 KB | Gam_L 512 B | dU (64 x 32) | dO (64 x 32)
    static constexpr uint32_t kA = 0, kKI = 32768, kGL = 49152;
    static constexpr uint32_t kDU = 50176;              // B operand rows 0-63 ...
    static constexpr uint32_t kDO = kDU + 64 * kRcVs * 2;   // ... and rows 64-127
    static constexpr uint32_t kStage = (kDO + 64 * kRcVs * 2 + 1023) / 1024 * 1024;
    static constexpr uint32_t kXB = kRcStages * kStage;     // bf16 dX, 128 x 32
    static constexpr uint32_t kBar = kXB + 128 * kRcVs * 2;
    static constexpr uint32_t kMisc = kBar + 16 * 8;
    static constexpr uint32_t kAlloc = kMisc + 16 + 1024;
    static_assert(kAlloc <= 232448, "shared memory budget exceeded");
    // TMEM: dU (M = 64 layout, 32 columns), acc[2]
    static constexpr uint32_t kTmDU = 0, kTmAcc = 32, kTmCols = 128;
};

struct RcParams {
    const unsigned char *packets;
    const float *dSf;        // [N, H, Dk, Dv] or null
    float *dS0;              // [N, H, Dk, Dv] or null
    float *dxs;              // [slots, Dk, Dv]: dX of every chunk
    const int32_t *cu, *chunk_off, *order;
    int32_t *status;
    long long slots;
    int N, T, H;
};

__global__ void __launch_bounds__(kRcThreads, 1)
rchain_kernel(const __grid_constant__ CUtensorMap tm_do, RcParams p) {
    using Ly = RcLayout;
    constexpr int VS = kRcVs;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(sm);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + Ly::kBar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + Ly::kMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + Ly::kMisc + 4);
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
    const int g0 = p.chunk_off[seq];
    if (g0 < 0 || ((long long)g0 + nchunks) * p.H > p.slots) {
        if (tid == 0) set_status(p.status, KDA_ERR_SEQLENS);
        return;
    }
    const size_t st_off = ((size_t)seq * p.H + h) * kDK * kDV + (size_t)vs * VS;

    if (tid == 0) {
        for (int i = 0; i < rbNum; ++i)
            mbar_init(&bars[i], (i == rbXbFull || i == rbDuFull) ? 4u : 1u);
        abort_flag[0] = 0;
        abort_flag[1] = 0;
        fence_mbar_init();
    }
    if (warp == 4 && lane == 0) prefetch_tmap(&tm_do);
    if (warp == 5) {
        tmem_alloc(tmem_slot, Ly::kTmCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // step i handles chunk j = nchunks - 1 - i
    auto packet = [&](int j) { return p.packets + ((size_t)(g0 + j) * p.H + h) * kPacketBytes; };
    auto stage = [&](int i) { return (uint32_t)(i % kRcStages) * Ly::kStage; };

    if (warp == 4) {
        // ------------------------------------------------------- loader
        int n_issued = 0;
        for (int i = 0; i < nchunks; ++i) {
            const int j = nchunks - 1 - i, s = i % kRcStages;
            bool ok = true;
            if (lane == 0 && i >= kRcStages)
                ok = wait_or_abort(&bars[rbFree + s], (i / kRcStages - 1) & 1, abort_flag, p.status);
            if (!__shfl_sync(0xffffffffu, ok, 0)) break;
            unsigned char *st = sm + stage(i);
            uint64_t *full = &bars[rbFull + s];
            if (lane == 0) mbar_arrive_expect_tx(full, 32768u + 16384u + 512u + 64u * VS * 2u);
            __syncwarp();
            if (lane < 2) bulk_load(st + Ly::kA + lane * 16384, packet(j) + lane * 16384, 16384, full);
            if (lane == 2) bulk_load(st + Ly::kKI, packet(j) + 32768, 16384, full);
            if (lane == 3) bulk_load(st + Ly::kGL, packet(j) + 65536, 512, full);
            if (lane == 4) tma_load_3d(st + Ly::kDO, &tm_do, full, vs * VS, h, t0 + j * kChunk);
            if (lane == 5 && i + kRcStages < nchunks)
                bulk_prefetch_l2(packet(j - kRcStages), (uint32_t)kPacketBytes);
            n_issued = i + 1;
        }
        if (lane == 0)
            for (int i = max(0, n_issued - kRcStages); i < n_issued; ++i)
                mbar_wait(&bars[rbFull + i % kRcStages], (i / kRcStages) & 1);
    } else if (warp == 5) {
        // ------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t kIdU = idesc_bf16(64, VS, 0, 1);    // Ki (K-major) x dX (MN-major)
            constexpr uint32_t kIdS = idesc_bf16(128, VS, 1, 1);   // [-W; Qe]^T (MN-major) x [dU; dO]
            const uint64_t d_xb = vs_desc<VS>(sbase + Ly::kXB, 128);
            // acc[i & 1] = [-W; Qe]^T rows 64-127 (the Qe rows) x dO: the half
            // that needs no dU, issued a step ahead
            auto issue_do = [&](int i) {
                const uint32_t st = sbase + stage(i);
                const uint64_t d_at = smem_desc(st + Ly::kA, 16384, 1024, kSw128);
                const uint64_t d_b = vs_desc<VS>(st + Ly::kDU, 128);
#pragma unroll
                for (int ks = 4; ks < 8; ++ks)
                    mma_bf16(tmem + Ly::kTmAcc + (uint32_t)(i & 1) * VS,
                             d_at + ((uint64_t)(ks * 2048) >> 4), d_b + vs_step<VS>(ks), kIdS, ks > 4);
            };
            bool ok = nchunks > 0 && spin_or_abort(&bars[rbFull], 0, abort_flag, p.status);
            if (ok) {
                tc_fence_after();
                issue_do(0);
            }
            for (int i = 0; i < nchunks && ok; ++i) {
                const uint32_t st = sbase + stage(i);
                if (!spin_or_abort(&bars[rbXbFull], i & 1, abort_flag, p.status)) break;
                tc_fence_after();
                {   // dU = Ki dX (M = 64)
                    const uint64_t d_ki = smem_desc(st + Ly::kKI, 16, 1024, kSw128);
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks)
                        mma_bf16(tmem + Ly::kTmDU, d_ki + kmaj_step(ks, 8192), d_xb + vs_step<VS>(ks),
                                 kIdU, ks > 0);
                }
                mma_commit(&bars[rbDuAcc]);
                if (!spin_or_abort(&bars[rbDuFull], i & 1, abort_flag, p.status)) break;
                tc_fence_after();
                {   // acc += [-W; Qe]^T rows 0-63 (the -W rows) x dU
                    const uint64_t d_at = smem_desc(st + Ly::kA, 16384, 1024, kSw128);
                    const uint64_t d_b = vs_desc<VS>(st + Ly::kDU, 128);
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        mma_bf16(tmem + Ly::kTmAcc + (uint32_t)(i & 1) * VS,
                                 d_at + ((uint64_t)(ks * 2048) >> 4), d_b + vs_step<VS>(ks), kIdS, 1);
                }
                mma_commit(&bars[rbDsAcc + (i & 1)]);
                mma_commit(&bars[rbFree + i % kRcStages]);
                if (i + 1 < nchunks) {
                    if (!spin_or_abort(&bars[rbFull + (i + 1) % kRcStages], ((i + 1) / kRcStages) & 1,
                                       abort_flag, p.status))
                        break;
                    tc_fence_after();
                    issue_do(i + 1);
                }
            }
            mma_commit(&bars[rbDrain]);
            mbar_wait(&bars[rbDrain], 0);
        }
    } else {
        // ------------------------------------------------------ chain warps
        const int c = tid, wq = warp;
        float dS[VS];
        {
            const float *src = p.dSf ? p.dSf + st_off + (size_t)c * kDV : nullptr;
#pragma unroll
            for (int jj = 0; jj < VS; jj += 4) {
                const float4 v = src ? *reinterpret_cast<const float4 *>(src + jj) : make_float4(0, 0, 0, 0);
                dS[jj] = v.x; dS[jj + 1] = v.y; dS[jj + 2] = v.z; dS[jj + 3] = v.w;
            }
        }
        const uint32_t xb = sbase + Ly::kXB;
        bool ok = true;
        for (int i = 0; i < nchunks && ok; ++i) {
            const int j = nchunks - 1 - i;
            const uint32_t st = sbase + stage(i);
            if (!spin_or_abort(&bars[rbFull + i % kRcStages], (i / kRcStages) & 1, abort_flag, p.status)) {
                ok = false;
                break;
            }
            // dX_j = Gam_L,j dS_{j+1}: kept for the assembly, and as bf16 operand
            const float g = reinterpret_cast<const float *>(sm + stage(i) + Ly::kGL)[c];
#pragma unroll
            for (int jj = 0; jj < VS; ++jj) dS[jj] *= g;
#pragma unroll
            for (int q8 = 0; q8 < VS / 8; ++q8)
                sts128(xb + vs_off<VS>(c, q8), pack2(dS[8 * q8], dS[8 * q8 + 1]),
                       pack2(dS[8 * q8 + 2], dS[8 * q8 + 3]), pack2(dS[8 * q8 + 4], dS[8 * q8 + 5]),
                       pack2(dS[8 * q8 + 6], dS[8 * q8 + 7]));
            fence_proxy_async();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[rbXbFull]);
            if (KDA_IN_RANGE(((long long)g0 + j) * p.H + h < p.slots, p.status)) {
                // fp32 dX_j for the assembly, off the chain: after the proxy fence
                float *dst = p.dxs + ((size_t)(g0 + j) * p.H + h) * kDK * kDV + (size_t)c * kDV +
                             (size_t)vs * VS;
#pragma unroll
                for (int jj = 0; jj < VS; jj += 4)
                    *reinterpret_cast<float4 *>(dst + jj) =
                        make_float4(dS[jj], dS[jj + 1], dS[jj + 2], dS[jj + 3]);
            }
            // dU (M = 64 accumulator: row r in TMEM lane 32 (r / 16) + r % 16)
            // -> bf16 rows 0-63 of the [dU; dO] operand
            if (!spin_or_abort(&bars[rbDuAcc], i & 1, abort_flag, p.status)) { ok = false; break; }
            tc_fence_after();
            {
                uint32_t v[32];
                tmem_ld32(tmem_addr(tmem, 32 * wq, Ly::kTmDU), v);
                tmem_wait_ld();
                if (lane < 16) {
                    const int r = 16 * wq + lane;
#pragma unroll
                    for (int e = 0; e < VS; e += 8)
                        sts128(st + Ly::kDU + vs_off<VS>(r, e / 8),
                               pack2(__uint_as_float(v[e]), __uint_as_float(v[e + 1])),
                               pack2(__uint_as_float(v[e + 2]), __uint_as_float(v[e + 3])),
                               pack2(__uint_as_float(v[e + 4]), __uint_as_float(v[e + 5])),
                               pack2(__uint_as_float(v[e + 6]), __uint_as_float(v[e + 7])));
                }
            }
            fence_proxy_async();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[rbDuFull]);
            // dS_j = dX_j + [-W; Qe]^T [dU; dO]
            if (!spin_or_abort(&bars[rbDsAcc + (i & 1)], (i >> 1) & 1, abort_flag, p.status)) {
                ok = false;
                break;
            }
            tc_fence_after();
            {
                uint32_t v[32];
                tmem_ld32(tmem_addr(tmem, 32 * wq, Ly::kTmAcc + (uint32_t)(i & 1) * VS), v);
                tmem_wait_ld();
#pragma unroll
                for (int jj = 0; jj < VS; ++jj) dS[jj] += __uint_as_float(v[jj]);
            }
        }
        if (ok && p.dS0) {
            float *dst = p.dS0 + st_off + (size_t)c * kDV;
#pragma unroll
            for (int jj = 0; jj < VS; jj += 4)
                *reinterpret_cast<float4 *>(dst + jj) = make_float4(dS[jj], dS[jj + 1], dS[jj + 2], dS[jj + 3]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (tid == 0) report_abort(abort_flag, p.status);
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem, Ly::kTmCols);
    }
}

// ============================================================ assembly
// Warp-level bf16 products (mma.sync m16n8k16, fp32 accumulation) over
// shared-memory tiles of bf16 rows (64 or 128 elements) whose 16-byte chunks
// are XOR-swizzled by row (chunk ^ (row & 7)), so ldmatrix reads of 8 rows
// hit 8 different bank groups.
struct Tile {
    uint32_t base;   // shared address (128-byte aligned)
    int rl;          // row length in elements
};
__device__ __forceinline__ uint32_t toff(const Tile &t, int r, int c) {
    return t.base + (uint32_t)(r * t.rl * 2) +
           ((((uint32_t)c >> 3) ^ ((uint32_t)r & 7u)) << 4) + (uint32_t)(c & 7) * 2u;
}
// acc (16 rows from m0, NT x 8 columns from n0) += A B over k in [kb, ke).
// A_T: A is stored transposed (rows = k); B_KN: B is stored k-major (rows =
// k), else n-major (rows = n).
template <int NT, bool A_T, bool B_KN>
__device__ __forceinline__ void wmma(float (&acc)[NT][4], const Tile &A, int m0, const Tile &B,
                                     int n0, int kb, int ke, int lane) {
    static_assert(NT % 2 == 0, "n tiles come in pairs");
    const int l7 = lane & 7, mi = lane >> 3;
#pragma unroll 2
    for (int k0 = kb; k0 < ke; k0 += 16) {
        uint32_t a[4];
        if (!A_T) ldsm_x4(toff(A, m0 + l7 + (mi & 1) * 8, k0 + (mi >> 1) * 8), a);
        else ldsm_x4_t(toff(A, k0 + l7 + (mi >> 1) * 8, m0 + (mi & 1) * 8), a);
#pragma unroll
        for (int n2 = 0; n2 < NT / 2; ++n2) {
            const int nb = n0 + 16 * n2;
            uint32_t b[4];
            if (!B_KN) ldsm_x4(toff(B, nb + l7 + (mi >> 1) * 8, k0 + (mi & 1) * 8), b);
            else ldsm_x4_t(toff(B, k0 + l7 + (mi & 1) * 8, nb + (mi >> 1) * 8), b);
            mma16816(acc[2 * n2], a, b[0], b[1]);
            mma16816(acc[2 * n2 + 1], a, b[2], b[3]);
        }
    }
}
template <int NT>
__device__ __forceinline__ void zero(float (&acc)[NT][4]) {
#pragma unroll
    for (int i = 0; i < NT; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
}
__device__ __forceinline__ void st_bf16x2(uint32_t addr, float a, float b) {
    asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(pack2(a, b)) : "memory");
}
__device__ __forceinline__ float ld_bf16(uint32_t addr) {
    unsigned short x;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(x) : "r"(addr));
    return __uint_as_float((uint32_t)x << 16);
}
// acc element e of n-tile nt: row m0 + g + 8 (e >> 1), column n0 + 8 nt + 2 q + (e & 1)
template <int NT>
__device__ __forceinline__ void store_tile(const Tile &T, float (&acc)[NT][4], int m0, int n0,
                                           int lane, float scale) {
    const int g = lane >> 2, q = lane & 3;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int col = n0 + 8 * nt + 2 * q;
        st_bf16x2(toff(T, m0 + g, col), scale * acc[nt][0], scale * acc[nt][1]);
        st_bf16x2(toff(T, m0 + g + 8, col), scale * acc[nt][2], scale * acc[nt][3]);
    }
}

struct AsmParams {
    const __nv_bfloat16 *q, *k, *v, *la, *beta, *dout;
    const float *ckpt, *dxs;   // [slots, Dk, Dv]: S_j entering chunk j; dX_j
    const int32_t *cu, *chunk_off;
    float *dq, *dk, *dv, *dla, *dbeta;
    int32_t *status;
    long long slots;
    int N, T, H;
};

struct AsmLayout {
    static constexpr uint32_t kKG = 0, kQG = 16384, kKI = 32768;
    static constexpr uint32_t kSolve = 49152;            // sL | sT, later V | dO
    static constexpr uint32_t kV = 49152, kDO = 65536;
    static constexpr uint32_t kS = 90112;                // S (bf16 128 x 128); Gam, dG fp32 temps
    static constexpr uint32_t kX = 122880;               // dX (bf16 128 x 128); la temp; dT | M1 | dAf
    static constexpr uint32_t kDT = 122880, kM1 = 131072, kDAF = 139264;
    static constexpr uint32_t kTB = 155648, kT = 163840, kP = 172032;
    static constexpr uint32_t kR1 = 180224;              // -W, then dU
    static constexpr uint32_t kR2 = 196608;              // U, then dW
    static constexpr uint32_t kB = 212992;               // beta [64]
    static constexpr uint32_t kSdx = kB + 256;           // rowsum(S * dX) [128]
    static constexpr uint32_t kCol = kSdx + 512;         // [4][128] colsum(Ki * Y) partials
    static constexpr uint32_t kColT = kCol + 2048;       // [4][64] colsum(T * dTb) partials
    static constexpr uint32_t kRow = kColT + 1024;       // [2][64] rowsum(dA * A_full) partials
    static constexpr uint32_t kAlloc = kRow + 512 + 128;
    static_assert(kAlloc <= 232448, "shared memory budget exceeded");
    static_assert(kSolve + 2 * 64 * kLDL * 4 + 4 * 16 * 17 * 4 <= kS, "solve scratch");
};

constexpr int kAsmThreads = 256;

__global__ void __launch_bounds__(kAsmThreads, 1) assemble_kernel(AsmParams p) {
    using Ly = AsmLayout;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *sm = smem_raw + ((128u - (smem_u32(smem_raw) & 127u)) & 127u);
    const uint32_t sb = smem_u32(sm);
    const int t = threadIdx.x, w = t >> 5, lane = t & 31, g8 = lane >> 2, q4 = lane & 3;
    const long long total = (long long)p.chunk_off[p.N] * p.H;
    const long long m = blockIdx.x;
    if (total < 0 || total > p.slots || m >= total) return;
    const Item it = item_of(m, p.H, p.chunk_off, p.cu, p.N);
    const int h = it.h, c0 = it.c0;
    // rows past the token axis are never touched (the debug build checks it)
    const int L = KDA_IN_RANGE(it.L == 0 || (long long)it.c0 + it.L <= p.T, p.status) ? it.L : 0;
    const size_t H = (size_t)p.H;
    auto rowk = [&](int r) { return ((size_t)(c0 + r) * H + h) * kDK; };   // [T, H, 128] row start

    const Tile tKg{sb + Ly::kKG, 128}, tQg{sb + Ly::kQG, 128}, tKi{sb + Ly::kKI, 128};
    const Tile tV{sb + Ly::kV, 128}, tDO{sb + Ly::kDO, 128};
    const Tile tS{sb + Ly::kS, 128}, tX{sb + Ly::kX, 128};
    const Tile tTb{sb + Ly::kTB, 64}, tT{sb + Ly::kT, 64}, tP{sb + Ly::kP, 64};
    const Tile tR1{sb + Ly::kR1, 128}, tR2{sb + Ly::kR2, 128};
    const Tile tDT{sb + Ly::kDT, 64}, tM1{sb + Ly::kM1, 64}, tDAF{sb + Ly::kDAF, 64};
    float *sB = reinterpret_cast<float *>(sm + Ly::kB);
    float *sSdx = reinterpret_cast<float *>(sm + Ly::kSdx);
    float *sCol = reinterpret_cast<float *>(sm + Ly::kCol);
    float *sColT = reinterpret_cast<float *>(sm + Ly::kColT);
    float *sRow = reinterpret_cast<float *>(sm + Ly::kRow);
    float *sGam = reinterpret_cast<float *>(sm + Ly::kS);           // fp32 [64][128] temp
    __nv_bfloat16 *sLa = reinterpret_cast<__nv_bfloat16 *>(sm + Ly::kX);   // bf16 [64][128] temp
    float *sL = reinterpret_cast<float *>(sm + Ly::kSolve);
    float *sT = sL + 64 * kLDL;

    // tile ownership: 64 x 128 outputs: rows m0 .. m0 + 15, columns n0 .. n0 + 63;
    // 64 x 64 outputs: the same rows, columns n6 .. n6 + 31
    const int m0 = 16 * (w & 3), n0 = 64 * (w >> 2), n6 = 32 * (w >> 2);

    // ---------------------------------------------------------------- P0
    // log_alpha and beta; sT cleared (the inverse writes only its blocks)
    {   // 4 x 16 B per thread, all loads in flight before the stores
        uint4 x[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = t + u * kAsmThreads, r = i >> 4, c8 = (i & 15) * 8;
            x[u] = r < L ? __ldg(reinterpret_cast<const uint4 *>(p.la + rowk(r) + c8))
                         : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = t + u * kAsmThreads, r = i >> 4, c8 = (i & 15) * 8;
            *reinterpret_cast<uint4 *>(sLa + r * 128 + c8) = x[u];
        }
    }
    if (t < 64) sB[t] = t < L ? __bfloat162float(p.beta[(size_t)(c0 + t) * H + h]) : 0.f;
    for (int i = t; i < 64 * kLDL; i += kAsmThreads) sT[i] = 0.f;
    __syncthreads();
    if (t < 128) {   // Gam = exp(in-chunk cumulative log-decay), per channel
        float gsum = 0.f;
        bool bad = false;
        for (int r = 0; r < 64; ++r) {
            const float la = __bfloat162float(sLa[r * 128 + t]);
            bad |= !(la <= 0.f);
            gsum += la;
            sGam[r * 128 + t] = expf(gsum);
        }
        bad |= !(gsum >= -80.f);
        if (bad) set_status(p.status, KDA_ERR_DECAY);
    }
    __syncthreads();
    // Kg, Qg, Ki as bf16 tiles (rows past L are zero: k, q read as zero); the
    // global loads of all eight steps are issued before any store
    {
        uint2 kk[8], qq[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int i = t + u * kAsmThreads, r = i >> 5, c4 = (i & 31) * 4;
            kk[u] = r < L ? __ldg(reinterpret_cast<const uint2 *>(p.k + rowk(r) + c4)) : make_uint2(0, 0);
            qq[u] = r < L ? __ldg(reinterpret_cast<const uint2 *>(p.q + rowk(r) + c4)) : make_uint2(0, 0);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int i = t + u * kAsmThreads, r = i >> 5, c4 = (i & 31) * 4;
            const float kv[4] = {bf16lo(kk[u].x), bf16hi(kk[u].x), bf16lo(kk[u].y), bf16hi(kk[u].y)};
            const float qv[4] = {bf16lo(qq[u].x), bf16hi(qq[u].x), bf16lo(qq[u].y), bf16hi(qq[u].y)};
            const float4 ga = *reinterpret_cast<const float4 *>(sGam + r * 128 + c4);
            const float gm[4] = {ga.x, ga.y, ga.z, ga.w};
#pragma unroll
            for (int e = 0; e < 4; e += 2) {
                st_bf16x2(toff(tKg, r, c4 + e), kv[e] * gm[e], kv[e + 1] * gm[e + 1]);
                st_bf16x2(toff(tQg, r, c4 + e), qv[e] * gm[e], qv[e + 1] * gm[e + 1]);
                st_bf16x2(toff(tKi, r, c4 + e), kv[e] / gm[e], kv[e + 1] / gm[e + 1]);
            }
        }
    }
    // Gam at this thread's accumulator positions (64 x 128 layout)
    float gam[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e)
            gam[nt][e] = sGam[(m0 + g8 + 8 * (e >> 1)) * 128 + n0 + 8 * nt + 2 * q4 + (e & 1)];
    __syncthreads();

    // ---------------------------------------------------------------- P1
    // A_full = Kg Ki^T and P = lower_incl(Qg Ki^T), 64 x 64
    float afull[4][4];
    {
        float pm[4][4];
        zero(afull);
        zero(pm);
        wmma<4, false, false>(afull, tKg, m0, tKi, n6, 0, 128, lane);
        wmma<4, false, false>(pm, tQg, m0, tKi, n6, 0, 128, lane);
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int r = m0 + g8 + 8 * (e >> 1), s = n6 + 8 * nt + 2 * q4 + (e & 1);
                afull[nt][e] = s < r ? afull[nt][e] : 0.f;
                sL[r * kLDL + s] = sB[r] * afull[nt][e];
                pm[nt][e] = s <= r ? pm[nt][e] : 0.f;
            }
        store_tile<4>(tP, pm, m0, n6, lane, 1.f);
    }
    __syncthreads();

    // ---------------------------------------------------------------- P2
    // warps 0-3: T = (I + L)^{-1}; warps 4-7: S_j and dX_j as bf16 tiles and
    // rowsum(S * dX), one row per warp and step
    if (w < 4) {
        invert_unit_lower(w, lane, sL, sT, 1);
    } else {
        const float *Sg = p.ckpt + (size_t)m * kDK * kDV;
        const float *Xg = p.dxs + (size_t)m * kDK * kDV;
        // rows w - 4 + 4 i, eight rows (16 loads of 16 B) in flight per batch
        for (int r0 = w - 4; r0 < 128; r0 += 32) {
            float4 a[8], b[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                a[u] = __ldg(reinterpret_cast<const float4 *>(Sg + (size_t)(r0 + 4 * u) * kDV + 4 * lane));
                b[u] = __ldg(reinterpret_cast<const float4 *>(Xg + (size_t)(r0 + 4 * u) * kDV + 4 * lane));
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int r = r0 + 4 * u;
                st_bf16x2(toff(tS, r, 4 * lane), a[u].x, a[u].y);
                st_bf16x2(toff(tS, r, 4 * lane + 2), a[u].z, a[u].w);
                st_bf16x2(toff(tX, r, 4 * lane), b[u].x, b[u].y);
                st_bf16x2(toff(tX, r, 4 * lane + 2), b[u].z, b[u].w);
                float d = a[u].x * b[u].x + a[u].y * b[u].y + a[u].z * b[u].z + a[u].w * b[u].w;
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
                if (lane == 0) sSdx[r] = d;
            }
        }
    }
    __syncthreads();
    // T in registers (64 x 64 layout); bf16 T and Tb = T diag(b); V and dO tiles
    float tr[4][4];
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int r = m0 + g8 + 8 * (e >> 1), s = n6 + 8 * nt + 2 * q4 + (e & 1);
            tr[nt][e] = s < r ? sT[r * kLDL + s] : (s == r ? 1.f : 0.f);
        }
    __syncthreads();   // sT read: the solve scratch becomes V and dO
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
        const int r = m0 + g8, s = n6 + 8 * nt + 2 * q4;
        st_bf16x2(toff(tT, r, s), tr[nt][0], tr[nt][1]);
        st_bf16x2(toff(tT, r + 8, s), tr[nt][2], tr[nt][3]);
        st_bf16x2(toff(tTb, r, s), tr[nt][0] * sB[s], tr[nt][1] * sB[s + 1]);
        st_bf16x2(toff(tTb, r + 8, s), tr[nt][2] * sB[s], tr[nt][3] * sB[s + 1]);
    }
    {
        uint2 vv[8], oo[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int i = t + u * kAsmThreads, r = i >> 5, c4 = (i & 31) * 4;
            vv[u] = r < L ? __ldg(reinterpret_cast<const uint2 *>(p.v + rowk(r) + c4)) : make_uint2(0, 0);
            oo[u] = r < L ? __ldg(reinterpret_cast<const uint2 *>(p.dout + rowk(r) + c4)) : make_uint2(0, 0);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int i = t + u * kAsmThreads, r = i >> 5, c4 = (i & 31) * 4;
            asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(toff(tV, r, c4)), "r"(vv[u].x),
                         "r"(vv[u].y)
                         : "memory");
            asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(toff(tDO, r, c4)), "r"(oo[u].x),
                         "r"(oo[u].y)
                         : "memory");
        }
    }
    __syncthreads();

    float acc[8][4];
    // ---------------------------------------------------------------- P3: -W = -Tb Kg
    zero(acc);
    wmma<8, false, true>(acc, tTb, m0, tKg, n0, 0, 64, lane);
    store_tile<8>(tR1, acc, m0, n0, lane, -1.f);
    __syncthreads();
    // ---------------------------------------------------------------- P4: U = Tb V + (-W) S
    zero(acc);
    wmma<8, false, true>(acc, tTb, m0, tV, n0, 0, 64, lane);
    wmma<8, false, true>(acc, tR1, m0, tS, n0, 0, 128, lane);
    store_tile<8>(tR2, acc, m0, n0, lane, 1.f);
    __syncthreads();
    // ---------------------------------------------------------------- P5: dU = P^T dO + Ki dX
    zero(acc);
    wmma<8, true, true>(acc, tP, m0, tDO, n0, 0, 64, lane);
    wmma<8, false, true>(acc, tKi, m0, tX, n0, 0, 128, lane);
    store_tile<8>(tR1, acc, m0, n0, lane, 1.f);
    __syncthreads();
    // ---------------------------------------------------------------- P6
    // dP = lower_incl(dO U^T); Y = U dX^T starts dKi; colsum(Ki * Y)
    float dki[8][4];
    {
        float dp[4][4];
        zero(dp);
        wmma<4, false, false>(dp, tDO, m0, tR2, n6, 0, 128, lane);
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int r = m0 + g8 + 8 * (e >> 1), s = n6 + 8 * nt + 2 * q4 + (e & 1);
                if (s > r) dp[nt][e] = 0.f;
            }
        zero(dki);
        wmma<8, false, false>(dki, tR2, m0, tX, n0, 0, 128, lane);
        __syncthreads();   // P read (P5) is done: dP takes its tile
        store_tile<4>(tP, dp, m0, n6, lane, 1.f);
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int e2 = 0; e2 < 2; ++e2) {
                const int col = n0 + 8 * nt + 2 * q4 + e2;
                float cs = ld_bf16(toff(tKi, m0 + g8, col)) * dki[nt][e2] +
                           ld_bf16(toff(tKi, m0 + g8 + 8, col)) * dki[nt][2 + e2];
#pragma unroll
                for (int o = 4; o <= 16; o <<= 1) cs += __shfl_xor_sync(0xffffffffu, cs, o);
                if (g8 == 0) sCol[(w & 3) * 128 + col] = cs;
            }
    }
    __syncthreads();
    // ---------------------------------------------------------------- P7: dKi += dP^T Qg
    wmma<8, true, true>(dki, tP, m0, tQg, n0, 0, 64, lane);
    // ---------------------------------------------------------------- P8: dQg = dO S^T + dP Ki
    float dg[8][4];
    zero(acc);
    wmma<8, false, false>(acc, tDO, m0, tS, n0, 0, 128, lane);
    wmma<8, false, true>(acc, tP, m0, tKi, n0, 0, 64, lane);
    {
        uint32_t qq[8][2];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int e2 = 0; e2 < 2; ++e2) {
                const int r = m0 + g8 + 8 * e2;
                qq[nt][e2] = r < L ? __ldg(reinterpret_cast<const unsigned int *>(
                                         p.q + rowk(r) + n0 + 8 * nt + 2 * q4))
                                   : 0u;
            }
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int e2 = 0; e2 < 2; ++e2) {
                const int r = m0 + g8 + 8 * e2;
                const int col = n0 + 8 * nt + 2 * q4;
                const float qv0 = bf16lo(qq[nt][e2]), qv1 = bf16hi(qq[nt][e2]);
                if (r < L)
                    *reinterpret_cast<float2 *>(p.dq + rowk(r) + col) =
                        make_float2(acc[nt][2 * e2] * gam[nt][2 * e2],
                                    acc[nt][2 * e2 + 1] * gam[nt][2 * e2 + 1]);
                dg[nt][2 * e2] = acc[nt][2 * e2] * qv0 * gam[nt][2 * e2];
                dg[nt][2 * e2 + 1] = acc[nt][2 * e2 + 1] * qv1 * gam[nt][2 * e2 + 1];
            }
    }
    // ---------------------------------------------------------------- P9: dW = -dU S^T
    zero(acc);
    wmma<8, false, false>(acc, tR1, m0, tS, n0, 0, 128, lane);
    store_tile<8>(tR2, acc, m0, n0, lane, -1.f);
    __syncthreads();
    // ---------------------------------------------------------------- P10
    // dTb = dU V^T + dW Kg^T; dT = dTb diag(b); colsum(T * dTb)
    {
        float dtb[4][4];
        zero(dtb);
        wmma<4, false, false>(dtb, tR1, m0, tV, n6, 0, 128, lane);
        wmma<4, false, false>(dtb, tR2, m0, tKg, n6, 0, 128, lane);
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int e2 = 0; e2 < 2; ++e2) {
                const int s = n6 + 8 * nt + 2 * q4 + e2;
                float cs = tr[nt][e2] * dtb[nt][e2] + tr[nt][2 + e2] * dtb[nt][2 + e2];
#pragma unroll
                for (int o = 4; o <= 16; o <<= 1) cs += __shfl_xor_sync(0xffffffffu, cs, o);
                if (g8 == 0) sColT[(w & 3) * 64 + s] = cs;
                dtb[nt][e2] *= sB[s];
                dtb[nt][2 + e2] *= sB[s];
            }
        store_tile<4>(tDT, dtb, m0, n6, lane, 1.f);
    }
    // ---------------------------------------------------------------- P11: dV = Tb^T dU, dKg = Tb^T dW
    zero(acc);
    wmma<8, true, true>(acc, tTb, m0, tR1, n0, 0, 64, lane);
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e2 = 0; e2 < 2; ++e2) {
            const int r = m0 + g8 + 8 * e2;
            if (r < L)
                *reinterpret_cast<float2 *>(p.dv + rowk(r) + n0 + 8 * nt + 2 * q4) =
                    make_float2(acc[nt][2 * e2], acc[nt][2 * e2 + 1]);
        }
    float dkg[8][4];
    zero(dkg);
    wmma<8, true, true>(dkg, tTb, m0, tR2, n0, 0, 64, lane);
    __syncthreads();   // dT written
    // ---------------------------------------------------------------- P12
    // M1 = T^T dT;  dA = strict_lower(-M1 T^T);  dAf = diag(b) dA;  rowsum(dA * A_full)
    {
        float m1[4][4];
        zero(m1);
        wmma<4, true, true>(m1, tT, m0, tDT, n6, 0, 64, lane);
        store_tile<4>(tM1, m1, m0, n6, lane, 1.f);
    }
    __syncthreads();
    {
        float da[4][4];
        zero(da);
        wmma<4, false, false>(da, tM1, m0, tT, n6, 0, 64, lane);
        float rs[2] = {0.f, 0.f};
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int r = m0 + g8 + 8 * (e >> 1), s = n6 + 8 * nt + 2 * q4 + (e & 1);
                const float d = s < r ? -da[nt][e] : 0.f;
                rs[e >> 1] += d * afull[nt][e];
                da[nt][e] = sB[r] * d;
            }
#pragma unroll
        for (int e2 = 0; e2 < 2; ++e2) {
            float x = rs[e2];
            x += __shfl_xor_sync(0xffffffffu, x, 1);
            x += __shfl_xor_sync(0xffffffffu, x, 2);
            if (q4 == 0) sRow[(w >> 2) * 64 + m0 + g8 + 8 * e2] = x;
        }
        store_tile<4>(tDAF, da, m0, n6, lane, 1.f);
    }
    __syncthreads();
    // ---------------------------------------------------------------- P13
    // dKg += dAf Ki;  dKi += dAf^T Kg
    wmma<8, false, true>(dkg, tDAF, m0, tKi, n0, 0, 64, lane);
    wmma<8, true, true>(dki, tDAF, m0, tKg, n0, 0, 64, lane);
    // ---------------------------------------------------------------- P14
    // dK = dKg Gam + dKi / Gam; dG = dKg Kg + dQg Qg - dKi Ki into the S region
    float *sdG = reinterpret_cast<float *>(sm + Ly::kS);
    uint32_t kk[8][2];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e2 = 0; e2 < 2; ++e2) {
            const int r = m0 + g8 + 8 * e2;
            kk[nt][e2] = r < L ? __ldg(reinterpret_cast<const unsigned int *>(
                                     p.k + rowk(r) + n0 + 8 * nt + 2 * q4))
                               : 0u;
        }
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e2 = 0; e2 < 2; ++e2) {
            const int r = m0 + g8 + 8 * e2;
            const int col = n0 + 8 * nt + 2 * q4;
            const float kv[2] = {bf16lo(kk[nt][e2]), bf16hi(kk[nt][e2])};
            float dkv[2], dgv[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int i = 2 * e2 + e;
                const float gm = gam[nt][i], ig = 1.f / gm;
                dkv[e] = dkg[nt][i] * gm + dki[nt][i] * ig;
                dgv[e] = dg[nt][i] + dkg[nt][i] * kv[e] * gm - dki[nt][i] * kv[e] * ig;
            }
            if (r < L)
                *reinterpret_cast<float2 *>(p.dk + rowk(r) + col) = make_float2(dkv[0], dkv[1]);
            *reinterpret_cast<float2 *>(sdG + r * 128 + col) = make_float2(dgv[0], dgv[1]);
        }
    __syncthreads();
    if (t < 128) {
        // dG of the last row also gets rowsum(X * dX) = rowsum(S * dX) + colsum(Ki * Y);
        // dlog_alpha = reverse cumulative sum of dG over the rows
        const float last = sSdx[t] + ((sCol[t] + sCol[128 + t]) + (sCol[256 + t] + sCol[384 + t]));
        float run = 0.f;
        for (int r = 63; r >= 0; --r) {
            run += sdG[r * 128 + t];
            if (r == L - 1) run += last;
            if (r < L) p.dla[rowk(r) + t] = run;
        }
    } else if (t < 192) {
        const int r = t - 128;
        if (r < L)
            p.dbeta[(size_t)(c0 + r) * H + h] =
                ((sColT[r] + sColT[64 + r]) + (sColT[128 + r] + sColT[192 + r])) +
                (sRow[r] + sRow[64 + r]);
    }
}

}  // namespace

// Reverse chain and assembly, after the forward's two passes have left the
// packets (workspace) and every chunk's entering state in a.ckpt.
cudaError_t launch_backward_tc(const BackwardTcArgs &a, cudaStream_t s) {
    if (a.N == 0 || a.T == 0) return cudaSuccess;
    CUtensorMap mdo;
    if (!make_tmap_bf16_3d(&mdo, a.d_out, a.T, a.H, kDV, kRcVs, kRcVs * 2))
        return cudaErrorInvalidValue;
    RcParams rp;
    rp.packets = a.packets;
    rp.dSf = a.dS_final;
    rp.dS0 = a.dS0;
    rp.dxs = a.dxs;
    rp.cu = a.cu_seqlens;
    rp.chunk_off = a.chunk_off;
    rp.order = a.order;
    rp.status = a.status;
    rp.slots = (long long)a.packet_slots;
    rp.N = a.N;
    rp.T = a.T;
    rp.H = a.H;
    cudaError_t e = cudaFuncSetAttribute(rchain_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)RcLayout::kAlloc);
    if (e != cudaSuccess) return e;
    const unsigned grid1 = (unsigned)a.N * a.H * (kDV / kRcVs);
    rchain_kernel<<<grid1, kRcThreads, RcLayout::kAlloc, s>>>(mdo, rp);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    AsmParams ap;
    ap.q = static_cast<const __nv_bfloat16 *>(a.q);
    ap.k = static_cast<const __nv_bfloat16 *>(a.k);
    ap.v = static_cast<const __nv_bfloat16 *>(a.v);
    ap.la = static_cast<const __nv_bfloat16 *>(a.log_alpha);
    ap.beta = static_cast<const __nv_bfloat16 *>(a.beta);
    ap.dout = static_cast<const __nv_bfloat16 *>(a.d_out);
    ap.ckpt = a.ckpt;
    ap.dxs = a.dxs;
    ap.cu = a.cu_seqlens;
    ap.chunk_off = a.chunk_off;
    ap.dq = a.dq;
    ap.dk = a.dk;
    ap.dv = a.dv;
    ap.dla = a.dla;
    ap.dbeta = a.dbeta;
    ap.status = a.status;
    ap.slots = (long long)a.packet_slots;
    ap.N = a.N;
    ap.T = a.T;
    ap.H = a.H;
    if ((e = cudaFuncSetAttribute(assemble_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)AsmLayout::kAlloc)) != cudaSuccess)
        return e;
    assemble_kernel<<<(unsigned)a.packet_slots, kAsmThreads, AsmLayout::kAlloc, s>>>(ap);
    return cudaGetLastError();
}

}  // namespace kda
