// kda_tc_common.cuh -- key-side building blocks shared by the tensor-core
// prefill kernels: gate prep (Qg, Kg, Ki, Gam_L over one 64-token chunk),
// the unit-lower-triangular inverse (Tb, masked P) and the -W operand.
//
// Tile layouts (shared memory, 128-byte swizzle, K-major rows of 64 channels):
//   KQ stage  [katom 0..1][Kg/-W rows 0..63 | Qg rows 0..63]   2 x 16 KB
//   KI stage  [katom 0..1][Ki rows 0..63]                       2 x 8 KB
//   TP stage  Tb rows 0..63 | zero rows 64..127 | P rows 128..191 (24 KB)
// and in TMEM: D_AP (lanes 0-63 = A, lanes 64-127 = P, 64 columns) and D_W
// (lanes 0-63 = W, 128 columns).
#pragma once

#include "kda_internal.cuh"
#include "sm100.cuh"

namespace kda {
namespace tc {

using namespace sm100;

constexpr int kDK = 128;           // key width handled by the tensor-core kernels
constexpr int kDV = 128;           // value width handled by the tensor-core kernels
constexpr int kLDL = 68;           // fp32 row stride of the solve scratch
constexpr int kPrepThreads = 256;  // threads running prep_chunk
constexpr int kSolveThreads = 128; // threads running solve_chunk (4 warps, lane quarters 0..3)
constexpr float kLog2e = 1.4426950408889634f;

// Bounded waits.  A wait that outlasts 2 s gives up: it raises the CTA's
// abort flag (abort_flag[0], so every role winds down) and notes where it
// gave up in abort_flag[1] (the barrier's shared-memory offset | thread index
// << 16).  Thread 0 reports both after the kernel's last barrier
// (report_abort): KDA_ERR_TIMEOUT in the status word, the note in status[8]
// and the block index in status[9].  Keeping the failure path out of the
// waits keeps the many call sites of a warp-specialised kernel small in the
// instruction cache.
__device__ __forceinline__ void raise_abort(volatile int *abort_flag, const uint64_t *bar) {
    abort_flag[1] = (int)((smem_u32(bar) & 0xFFFFu) | ((uint32_t)threadIdx.x << 16));
    abort_flag[0] = 1;
}
__device__ __forceinline__ void report_abort(const volatile int *abort_flag, int32_t *status) {
    if (!abort_flag[0]) return;
    set_status(status, KDA_ERR_TIMEOUT);
    if (status && atomicCAS(status + 8, 0, abort_flag[1]) == 0) status[9] = (int32_t)blockIdx.x;
}

// Waiting threads stay suspended in try_wait (no issue slots taken from
// working warps) and wake when the phase completes.
__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity,
                                              volatile int *abort_flag, int32_t *) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t start = globaltimer_ns();
#pragma unroll 1
    for (;;) {
        if (mbar_try_wait_sleep(bar, parity, 20000u)) return true;
        if (*abort_flag) return false;
        if (globaltimer_ns() - start > 2000000000ull) break;
    }
    raise_abort(abort_flag, bar);
    return false;
}

// Polls instead of suspending: for the few threads on a latency-critical
// chain, where the wake-up of a suspended waiter costs hundreds of cycles.
__device__ __forceinline__ bool spin_or_abort(uint64_t *bar, uint32_t parity,
                                              volatile int *abort_flag, int32_t *) {
    uint64_t start = 0;
#pragma unroll 1
    for (uint32_t n = 1;; ++n) {
        if (mbar_test_wait(bar, parity)) return true;
        if ((n & 1023u) == 0) {
            if (*abort_flag) return false;
            const uint64_t now = globaltimer_ns();
            if (start == 0) start = now;
            else if (now - start > 2000000000ull) break;
        }
    }
    raise_abort(abort_flag, bar);
    return false;
}

// Maps item index m (= global chunk g * H + head) to its chunk.
struct Item {
    int h, c0, L;
    int m;   // packet index m; negative: this CTA has no further item
};
static __device__ __noinline__ Item item_of(long long m, int H, const int32_t *chunk_off,
                                        const int32_t *cu, int N) {
    const int g = (int)(m / H);
    Item it;
    it.m = (int)m;
    it.h = (int)(m % H);
    int lo = 0, hi = N;   // largest n with chunk_off[n] <= g
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (chunk_off[mid] <= g) lo = mid;
        else hi = mid;
    }
    // 64-bit: with saturated offsets (overlapping sequences) j can exceed
    // the sequence's chunk count; such an item gets no rows (L = 0).
    const long long c0 = (long long)cu[lo] + (long long)(g - chunk_off[lo]) * kChunk;
    const long long L = (long long)cu[lo + 1] - c0;
    if (c0 < 0 || c0 > 0x7fffffffLL || L <= 0) {
        it.c0 = 0;
        it.L = 0;
    } else {
        it.c0 = (int)c0;
        it.L = (int)(L < kChunk ? L : kChunk);
    }
    return it;
}

// 16-byte shared store / load helpers
__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                       uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
                 "r"(d)
                 : "memory");
}
__device__ __forceinline__ void sts16(uint32_t addr, uint16_t a) {
    asm volatile("st.shared.b16 [%0], %1;" ::"r"(addr), "h"(a) : "memory");
}
__device__ __forceinline__ uint16_t bf16_bits(float x) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}
__device__ __forceinline__ void sts32(uint32_t addr, uint32_t a) {
    asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(a) : "memory");
}
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi) { return pack_bf16(lo, hi); }

// Byte offset of 16-byte chunk `chunk` of row `row` in a VS-wide (32 or 64)
// MN-major tile.
template <int VS>
__device__ __forceinline__ uint32_t vs_off(uint32_t row, uint32_t chunk, uint32_t = 0) {
    static_assert(VS == 32 || VS == 64, "narrow value slices only");
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

// ---------------------------------------------------------------------------
// Gate prep for one chunk, run by kPrepThreads threads (t = 0..255) that
// synchronise on named barrier `bar_id`.  On entry the KQ stage holds raw k
// (rows 0-63) and q (rows 64-127) and the KI stage raw log_alpha, as the TMA
// left them.  On exit (after a proxy fence) they hold Kg, Qg and Ki; rows at
// or past L are zero.  sGL_s receives Gam_L (128 channels), sB_s beta (64
// rows, zero past L).  sGP / sSUF are [16][128] fp32 scratch; with
// kScratchInKI they are the two 8 KB halves of the KI stage itself, free once
// every raw log_alpha has been read (one more barrier) and overwritten by Ki.
//
// alpha = 2^(log_alpha log2 e) once per element; Gam_r is the running product
// of alpha inside the chunk and 1/Gam_r = (1/Gam_L) prod_{j>r} alpha_j, so no
// element needs a second exponential or a division.
//
// The factorisation needs every log_alpha <= 0 (finite) and every channel's
// Gam_L >= exp(-80); a chunk that breaks either records KDA_ERR_DECAY in
// `status` (its chain's results are then unspecified; nothing else changes).
// ---------------------------------------------------------------------------
template <bool kScratchInKI = false>
__device__ __forceinline__ void prep_chunk(int t, uint32_t kq_stage, uint32_t ki_stage,
                                           float *sGP, float *sSUF, float *sGL_s, float *sB_s,
                                           const __nv_bfloat16 *beta, int c0, int L, int H, int h,
                                           uint32_t bar_id, int32_t *status) {
    const int cg = t & 15, rg = t >> 4;   // 8-channel group, 4-row group
    const int a = cg >> 3, ch = cg & 7;
    const uint32_t kq = kq_stage + a * 16384;
    const uint32_t ki = ki_stage + a * 8192;
    // beta comes from global memory: start its load before anything else
    float beta_r = 0.f;
    if (t >= 128 && t < 128 + kChunk && t - 128 < L)
        beta_r = __bfloat162float(beta[(size_t)(c0 + t - 128) * H + h]);
    // pass 0: alpha; in-group prefix and suffix products
    float pre[4][8], suf[4][8];
    bool bad = false;   // a log_alpha above 0 or not finite
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = rg * 4 + i;
        uint4 raw = lds128(ki + sw128_off(r, ch));
        if (r >= L) raw = make_uint4(0, 0, 0, 0);  // past the end: alpha = 1
        const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float la = (e & 1) ? bf16hi(w4[e >> 1]) : bf16lo(w4[e >> 1]);
            bad |= !(la <= 0.f);
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
    if (kScratchInKI) named_bar(bar_id, kPrepThreads);   // every log_alpha read before sGP lands on it
    {
        float *gpp = sGP + rg * 128 + cg * 8;
        *reinterpret_cast<float4 *>(gpp) = make_float4(pre[3][0], pre[3][1], pre[3][2], pre[3][3]);
        *reinterpret_cast<float4 *>(gpp + 4) = make_float4(pre[3][4], pre[3][5], pre[3][6], pre[3][7]);
    }
    named_bar(bar_id, kPrepThreads);
    // scan over the 16 row groups, one thread per channel:
    // sGP <- exclusive prefix, sSUF <- (1/Gam_L) exclusive suffix, sGL <- Gam_L
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
        sGL_s[t] = px;
        bad |= !(px >= kMinChunkDecay);   // also catches a NaN product
        float sx = rcp_approx(px);   // 1/Gam_L, once per channel
#pragma unroll
        for (int g = 15; g >= 0; --g) {
            sSUF[g * 128 + t] = sx;
            sx *= gv[g];
        }
    } else if (t < 128 + kChunk) {
        sB_s[t - 128] = beta_r;
    }
    named_bar(bar_id, kPrepThreads);
    if (__any_sync(0xffffffffu, bad) && (t & 31) == 0) set_status(status, KDA_ERR_DECAY);
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
    // the next chunk's pass 0 (or, with kScratchInKI, this chunk's Ki)
    // overwrites sGP and sSUF: everyone must have read them
    named_bar(bar_id, kPrepThreads);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = rg * 4 + i;
        uint32_t gb[4], gib[4];
#pragma unroll
        for (int e2 = 0; e2 < 4; ++e2) {
            gb[e2] = pack2(ef[2 * e2] * pre[i][2 * e2], ef[2 * e2 + 1] * pre[i][2 * e2 + 1]);
            gib[e2] = pack2(ci[2 * e2] * suf[i][2 * e2], ci[2 * e2 + 1] * suf[i][2 * e2 + 1]);
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
}

// ---------------------------------------------------------------------------
// Solve for one chunk, run by 4 warps (sw = 0..3 owns TMEM lanes 32 sw..) that
// synchronise on named barrier `bar_id`.  Reads D_AP from TMEM (column
// tm_ap), writes L = strict_lower(diag(b) A) to sL and the masked bf16 P as a
// 64-row K-major tile at `p_tile`, arrives once on `ap_free` when D_AP may be
// overwritten, then builds T = (I + L)^{-1} in sT (invert_unit_lower).
// Blocks of sT above the diagonal blocks must be zero on entry (they are
// never written).  write_tb() then turns T into the bf16 Tb tile.
// ---------------------------------------------------------------------------
// P = lower_incl(Q K^T) rows (TMEM lanes 64..127 of the A/P accumulator at
// column tm_ap) -> masked bf16 64-row K-major tile at `p_tile`.  Run by the
// solve warps with lane quarters 2 and 3 (sw = 2, 3); a no-op for sw < 2.
__device__ __forceinline__ void write_p(int sw, int lane, uint32_t tmem, uint32_t tm_ap,
                                       uint32_t p_tile) {
    if (sw < 2) return;
    const int r = 32 * (sw & 1) + lane;
#pragma unroll 1
    for (int j2 = 0; j2 < 8; j2 += 2) {
        uint32_t v[16];
        tmem_ld16(tmem_addr(tmem, 32 * sw, tm_ap + 8 * j2), v);
        tmem_wait_ld();
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
            uint32_t o[4];
#pragma unroll
            for (int e2 = 0; e2 < 4; ++e2) {
                const int cl = 8 * jj + 2 * e2, c = 8 * j2 + cl;
                const float x0 = (c <= r) ? __uint_as_float(v[cl]) : 0.f;
                const float x1 = (c + 1 <= r) ? __uint_as_float(v[cl + 1]) : 0.f;
                o[e2] = pack2(x0, x1);
            }
            sts128(p_tile + sw128_off(r, j2 + jj), o[0], o[1], o[2], o[3]);
        }
    }
}

// ---------------------------------------------------------------------------
// T = (I + L)^{-1} for a strictly lower 64 x 64 fp32 L in sL (row stride
// kLDL), run by 4 warps (sw = 0..3) that synchronise on named barrier
// `bar_id`.  With 16x16 blocks, D_i = (I + L_ii)^{-1} and M_ik = D_i L_ik:
//   phase 1: the four D_i by substitution (one block per warp, one column
//            per lane);
//   phase 2: the six M_ik (i > k), written over L_ik;
//   phase 3: block forward substitution T_ij = -sum_{j <= k < i} M_ik T_kj
//            (T_jj = D_j) by 8-column strips with mma.sync tf32.
// Scaling the blocks first keeps every step of the substitution one product
// whose operands are already in shared memory.  Blocks of sT above the
// diagonal must be zero on entry (they are never written); sL's off-diagonal
// blocks are overwritten.  On return each warp has written its strips (warps
// 0, 1: block column 0; warps 2, 3: block columns 1 and 2; D_3 since phase
// 1); the caller orders them before any other reader.
// ---------------------------------------------------------------------------
// acc += A_blk B_blk over one 16-wide k block: A rows 16 ai (row stride kLDL)
// from column 16 ak, B rows 16 ak .. from column c0 (an 8-column strip).
__device__ __forceinline__ void blk_mma(float (&acc)[4], const float *A, int ai, int ak,
                                        const float *B, int c0, int g, int tq) {
#pragma unroll
    for (int kk = 0; kk < 16; kk += 8) {
        const float *Ar = A + (16 * ai + g) * kLDL + 16 * ak + kk + tq;
        const uint32_t af[4] = {tf32_bits(Ar[0]), tf32_bits(Ar[8 * kLDL]), tf32_bits(Ar[4]),
                                tf32_bits(Ar[8 * kLDL + 4])};
        const float *Bc = B + (16 * ak + kk + tq) * kLDL + c0 + g;
        const uint32_t bfr[2] = {tf32_bits(Bc[0]), tf32_bits(Bc[4 * kLDL])};
        mma_tf32_16x8x8(acc, af, bfr);
    }
}
// C fragment (16 x 8) -> -C at rows 16 i of the strip at column c0 of sT
__device__ __forceinline__ void store_neg(float *sT, int i, int c0, const float (&d)[4], int g,
                                          int tq) {
    float *o = sT + (16 * i) * kLDL + c0;
    o[g * kLDL + 2 * tq] = -d[0];
    o[g * kLDL + 2 * tq + 1] = -d[1];
    o[(g + 8) * kLDL + 2 * tq] = -d[2];
    o[(g + 8) * kLDL + 2 * tq + 1] = -d[3];
}

__device__ __forceinline__ void invert_unit_lower(int sw, int lane, float *sL, float *sT,
                                                  uint32_t bar_id) {
    const int g = lane >> 2, tq = lane & 3;
    // phase 1: invert the four 16x16 diagonal blocks, one block per warp, one
    // column per lane (lanes 0-15)
    if (lane < 16) {
        const int o = 16 * sw, j = lane;
        float col[16];
#pragma unroll
        for (int aa = 0; aa < 16; ++aa) col[aa] = 0.f;
#pragma unroll
        for (int aa = 0; aa < 16; ++aa) {
            // four independent partial sums keep the dependent chain short
            float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
            for (int m4 = 0; m4 < aa; m4 += 4) {
                const float4 l = *reinterpret_cast<const float4 *>(sL + (o + aa) * kLDL + o + m4);
                a0 = fmaf(l.x, col[m4], a0);
                if (m4 + 1 < aa) a1 = fmaf(l.y, col[m4 + 1], a1);
                if (m4 + 2 < aa) a2 = fmaf(l.z, col[m4 + 2], a2);
                if (m4 + 3 < aa) a3 = fmaf(l.w, col[m4 + 3], a3);
            }
            col[aa] = (aa == j) ? 1.f : -((a0 + a1) + (a2 + a3));
        }
#pragma unroll
        for (int aa = 0; aa < 16; ++aa) sT[(o + aa) * kLDL + o + j] = col[aa];
    }
    named_bar(bar_id, kSolveThreads);

    // phase 2: M_ik = D_i L_ik for the six blocks below the diagonal, twelve
    // 8-column halves, three per warp: unit u -> block (i, k) and half h
    {
        float m[3][4];
#pragma unroll
        for (int v = 0; v < 3; ++v) {
            const int u = sw + 4 * v;                 // 0..11
            const int blk = u >> 1, h = u & 1;        // blocks (1,0) (2,0) (2,1) (3,0) (3,1) (3,2)
            const int i = blk < 1 ? 1 : blk < 3 ? 2 : 3;
            const int k = blk < 1 ? 0 : blk < 3 ? blk - 1 : blk - 3;
#pragma unroll
            for (int e = 0; e < 4; ++e) m[v][e] = 0.f;
            // D_i (rows and columns of block i in sT) times L_ik (rows of block i in sL)
#pragma unroll
            for (int kk = 0; kk < 16; kk += 8) {
                const float *Ar = sT + (16 * i + g) * kLDL + 16 * i + kk + tq;
                const uint32_t af[4] = {tf32_bits(Ar[0]), tf32_bits(Ar[8 * kLDL]), tf32_bits(Ar[4]),
                                        tf32_bits(Ar[8 * kLDL + 4])};
                const float *Bc = sL + (16 * i + kk + tq) * kLDL + 16 * k + 8 * h + g;
                const uint32_t bfr[2] = {tf32_bits(Bc[0]), tf32_bits(Bc[4 * kLDL])};
                mma_tf32_16x8x8(m[v], af, bfr);
            }
        }
        named_bar(bar_id, kSolveThreads);   // every L_ik read before M_ik lands on it
#pragma unroll
        for (int v = 0; v < 3; ++v) {
            const int u = sw + 4 * v;
            const int blk = u >> 1, h = u & 1;
            const int i = blk < 1 ? 1 : blk < 3 ? 2 : 3;
            const int k = blk < 1 ? 0 : blk < 3 ? blk - 1 : blk - 3;
            float *o = sL + (16 * i) * kLDL + 16 * k + 8 * h;
            o[g * kLDL + 2 * tq] = m[v][0];
            o[g * kLDL + 2 * tq + 1] = m[v][1];
            o[(g + 8) * kLDL + 2 * tq] = m[v][2];
            o[(g + 8) * kLDL + 2 * tq + 1] = m[v][3];
        }
        named_bar(bar_id, kSolveThreads);
    }

    // phase 3: each strip only reads M, the diagonal blocks and its own
    // columns, so a warp needs no barrier until Tb is written.  Products that
    // do not wait on the strip's latest block are issued a step early.
    const int q = sw & 1;
    if (sw < 2) {
        const int c0 = 8 * q;   // block column 0
        float t1[4] = {0.f, 0.f, 0.f, 0.f}, t2[4] = {0.f, 0.f, 0.f, 0.f},
              t3[4] = {0.f, 0.f, 0.f, 0.f};
        blk_mma(t1, sL, 1, 0, sT, c0, g, tq);
        blk_mma(t2, sL, 2, 0, sT, c0, g, tq);
        blk_mma(t3, sL, 3, 0, sT, c0, g, tq);
        store_neg(sT, 1, c0, t1, g, tq);
        __syncwarp();
        blk_mma(t2, sL, 2, 1, sT, c0, g, tq);
        blk_mma(t3, sL, 3, 1, sT, c0, g, tq);
        store_neg(sT, 2, c0, t2, g, tq);
        __syncwarp();
        blk_mma(t3, sL, 3, 2, sT, c0, g, tq);
        store_neg(sT, 3, c0, t3, g, tq);
        __syncwarp();
    } else {
        const int c1 = 16 + 8 * q, c2 = 32 + 8 * q;   // block columns 1 and 2
        float t21[4] = {0.f, 0.f, 0.f, 0.f}, t31[4] = {0.f, 0.f, 0.f, 0.f},
              t32[4] = {0.f, 0.f, 0.f, 0.f};
        blk_mma(t21, sL, 2, 1, sT, c1, g, tq);
        blk_mma(t31, sL, 3, 1, sT, c1, g, tq);
        blk_mma(t32, sL, 3, 2, sT, c2, g, tq);
        store_neg(sT, 2, c1, t21, g, tq);
        store_neg(sT, 3, c2, t32, g, tq);
        __syncwarp();
        blk_mma(t31, sL, 3, 2, sT, c1, g, tq);
        store_neg(sT, 3, c1, t31, g, tq);
        __syncwarp();
    }
}

// L = strict_lower(diag(b) A) from rows 0..63 of the A/P accumulator (TMEM
// column tm_ap) into sL, by the two warps owning TMEM lanes 0..63 (sw = 0, 1).
__device__ __forceinline__ void build_l(int sw, int lane, uint32_t tmem, uint32_t tm_ap, float *sL,
                                        const float *sB_s) {
    const int r = 32 * sw + lane;
    const float br = sB_s[r];
    float *Lr = sL + r * kLDL;
#pragma unroll 1
    for (int c0 = 0; c0 < 64; c0 += 16) {
        uint32_t v[16];
        tmem_ld16(tmem_addr(tmem, 32 * sw, tm_ap + c0), v);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 16; c += 4) {
            float4 w;
            w.x = (c0 + c + 0 < r) ? br * __uint_as_float(v[c]) : 0.f;
            w.y = (c0 + c + 1 < r) ? br * __uint_as_float(v[c + 1]) : 0.f;
            w.z = (c0 + c + 2 < r) ? br * __uint_as_float(v[c + 2]) : 0.f;
            w.w = (c0 + c + 3 < r) ? br * __uint_as_float(v[c + 3]) : 0.f;
            *reinterpret_cast<float4 *>(Lr + c0 + c) = w;
        }
    }
}

// kEarlyP: write P and release D_AP (one arrival on `ap_free`) right after
// reading L.  Otherwise P stays in TMEM: the caller writes it with write_p()
// and arrives on `ap_free` itself, later.
template <bool kEarlyP = true>
__device__ __forceinline__ void solve_chunk(int sw, int lane, uint32_t tmem, uint32_t tm_ap,
                                            uint32_t p_tile, float *sL, float *sT,
                                            const float *sB_s, uint64_t *ap_free,
                                            uint32_t bar_id) {
    const int t = sw * 32 + lane;
    if (sw < 2) {
        build_l(sw, lane, tmem, tm_ap, sL, sB_s);
    } else if (kEarlyP) {
        write_p(sw, lane, tmem, tm_ap, p_tile);
    }
    tc_fence_before();
    named_bar(bar_id, kSolveThreads);
    if (kEarlyP && t == 0) mbar_arrive(ap_free);

    invert_unit_lower(sw, lane, sL, sT, bar_id);
}

// Tb = T diag(b) -> bf16 into rows 0..63 of the K-major tile at `tp`, one
// 8-column chunk at a time: each warp writes the strips it computed in
// solve_chunk, and warps 0 and 1 also the two strips of block 3 (D_3, final
// since phase 1), so only the caller's own ordering is needed before it.
// Ends with a proxy fence and a barrier.
__device__ __forceinline__ void write_tb(int sw, int lane, uint32_t tp, const float *sT,
                                         const float *sB_s, uint32_t bar_id) {
    {
        const int q = sw & 1;
#pragma unroll
        for (int pass = 0; pass < 2; ++pass) {
            const int cb = sw < 2 ? (pass == 0 ? 0 : 3) : 1 + pass;
            const int ch = 2 * cb + q;
            const float4 b0 = *reinterpret_cast<const float4 *>(sB_s + 8 * ch);
            const float4 b1 = *reinterpret_cast<const float4 *>(sB_s + 8 * ch + 4);
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
                const int r = lane + 32 * rr;
                const float *Tr = sT + r * kLDL + 8 * ch;
                const float4 t0 = *reinterpret_cast<const float4 *>(Tr);
                const float4 t1 = *reinterpret_cast<const float4 *>(Tr + 4);
                sts128(tp + sw128_off(r, ch), pack2(t0.x * b0.x, t0.y * b0.y),
                       pack2(t0.z * b0.z, t0.w * b0.w), pack2(t1.x * b1.x, t1.y * b1.y),
                       pack2(t1.z * b1.z, t1.w * b1.w));
            }
        }
    }
    fence_proxy_async();
    named_bar(bar_id, kSolveThreads);
}

// ---------------------------------------------------------------------------
// W (TMEM column tm_w, lanes 0..63, fp32) -> -W as bf16 over the Kg rows of
// the KQ stage.  Run by the two warps owning TMEM lanes 0..63 (sw = 0, 1).
// Ends with the proxy and tcgen05 fences; the caller then arrives.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void convert_w(int sw, int lane, uint32_t tmem, uint32_t tm_w,
                                          uint32_t kq_stage) {
    const int r = 32 * sw + lane;
#pragma unroll
    for (int blk = 0; blk < 4; ++blk) {
        uint32_t v[32];
        tmem_ld32(tmem_addr(tmem, 32 * sw, tm_w + 32 * blk), v);
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
            sts128(kq_stage + aa * 16384 + sw128_off(r, chunk), o[0], o[1], o[2], o[3]);
        }
    }
    fence_proxy_async();
    tc_fence_before();
    __syncwarp();
}

}  // namespace tc
}  // namespace kda
