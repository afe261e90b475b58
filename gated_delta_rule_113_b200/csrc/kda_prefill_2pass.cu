// kda_prefill_2pass.cu -- two-pass tensor-core KDA prefill (bf16 I/O, fp32 state).
//
// The chunked evaluation of the recurrence of the page "Kimi K3: Open Frontier
// Intelligence and Implementation Framework" (section "Hybrid Attention
// Mechanism", KDA bullet) splits into work that depends only on one chunk's
// keys, queries and gates, and a short sequential state chain.  The key-side
// work dominates the latency of a chunk, so it runs in its own pass:
//
//   pass 1  (kside_kernel, persistent, one chunk x head per item, spread over
//           every SM): gate prep, [A;P] = [Kg;Qg] Ki^T, the triangular
//           inverse Tb, W = Tb Kg.  It writes one operand packet per item to
//           the workspace, in the exact shared-memory layout pass 2 consumes:
//             [-W;Qg] 32 KB | Ki 16 KB | Tb 8 KB | P 8 KB | Gam_L 512 B
//   pass 2  (chain_kernel, one CTA per (sequence, head, VS-wide value slice)):
//           streams the packets and the value tile with bulk copies and runs
//           only the value-side products and the fp32 state chain:
//             D1  = Tb V ; D1 += [-W;Qg] S  (U | Qg S) ; dS = Ki^T U ;
//             D1 += [0;P] U  (O) ;  S <- Diag(Gam_L) (S + dS)
//
// The packets cost ~1 KB of extra HBM traffic per token-head (written once,
// read once; the value slices of a chain share each packet through L2).
#include "kda_internal.cuh"
#include "kda_tc_common.cuh"
#include "sm100.cuh"

namespace kda {
namespace {

using namespace sm100;
using namespace tc;

// Optional per-chunk timeline of pass 2's CTA 0 (clock64 per pipeline event),
// compiled in only with -DKDA_TRACE for profiling builds; a no-op otherwise.
#ifdef KDA_TRACE
__device__ unsigned long long g_kda_trace1[64 * 16];
#define KDA_TRACE1(n, e)                                                          \
    do {                                                                          \
        if (blockIdx.x == 0 && (n) < 64) g_kda_trace1[(n) * 16 + (e)] = clock64(); \
    } while (0)
__device__ unsigned long long g_kda_trace2[64 * 16];
#define KDA_TRACE2(n, e)                                                          \
    do {                                                                          \
        if (blockIdx.x == 0 && (n) < 64) g_kda_trace2[(n) * 16 + (e)] = clock64(); \
    } while (0)
#else
#define KDA_TRACE1(n, e) \
    do {                 \
    } while (0)
#define KDA_TRACE2(n, e) \
    do {                 \
    } while (0)
#endif

// packet layout (bytes)
constexpr uint32_t kPkKQ = 0;
constexpr uint32_t kPkKI = 32768;
constexpr uint32_t kPkTb = 49152;
constexpr uint32_t kPkP = 57344;
constexpr uint32_t kPkGL = 65536;
static_assert(kPkGL + 512 <= kPacketBytes, "packet layout");

// Maps item index m (= global chunk g * H + head) to its chunk.
struct Item {
    int h, c0, L;
};
__device__ __forceinline__ Item item_of(long long m, int H, const int32_t *chunk_off,
                                        const int32_t *cu, int N) {
    const int g = (int)(m / H);
    Item it;
    it.h = (int)(m % H);
    int lo = 0, hi = N;   // largest n with chunk_off[n] <= g
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (chunk_off[mid] <= g) lo = mid;
        else hi = mid;
    }
    const int j = g - chunk_off[lo];
    it.c0 = cu[lo] + j * kChunk;
    it.L = min(kChunk, cu[lo + 1] - it.c0);
    return it;
}

// ============================================================ pass 1
constexpr int kKsWarps = 15;   // 0-7 prep, 8-11 solve, 12 TMA loads, 13 MMA, 14 packet stores
constexpr int kKsThreads = kKsWarps * 32;
enum KsRole { kKsPrep0 = 0, kKsSolve0 = 8, kKsTma = 12, kKsMma = 13, kKsStore = 14 };
enum KsBars {
    kbRawFull = 0,   // [2] TMA -> prep
    kbKqFull = 2,    // [2] count 8: prep -> MMA, stores (Qg, Ki, Gam_L final)
    kbApFull = 4,    // [2] MMA_AP -> solve
    kbApFree = 6,    // [2] solve read D_AP[s] -> MMA
    kbTbFull = 8,    // [2] solve -> MMA, stores (Tb, P final)
    kbWaccFull = 10, // MMA_W -> solve
    kbWReady = 11,   // [2] count 2: -W written -> MMA (D_W free), stores
    kbStored = 13,   // [2] every store of a stage has read shared memory -> TMA
    kbDrain = 15,
    kbNum = 16
};

struct KsLayout {
    static constexpr uint32_t kKQ = 0;                      // 2 x 32 KB
    static constexpr uint32_t kKI = kKQ + 2 * 32768;        // 2 x 16 KB
    static constexpr uint32_t kTP = kKI + 2 * 16384;        // 2 x 24 KB
    static constexpr uint32_t kL = kTP + 2 * 24576;
    static constexpr uint32_t kT = kL + 64 * kLDL * 4;
    static constexpr uint32_t kXw = kT + 64 * kLDL * 4;     // fp32 4 x [16][17]
    static constexpr uint32_t kGP = kXw + 4 * 16 * 17 * 4;
    static constexpr uint32_t kSUF = kGP + 16 * 128 * 4;
    static constexpr uint32_t kGL = kSUF + 16 * 128 * 4;    // [2][128]
    static constexpr uint32_t kB = kGL + 2 * 128 * 4;       // [2][64]
    static constexpr uint32_t kBar = kB + 2 * 64 * 4;
    static constexpr uint32_t kMisc = kBar + 16 * 8;
    static constexpr uint32_t kAlloc = kMisc + 16 + 1024;
    static_assert(kAlloc <= 232448, "shared memory budget exceeded");
    static constexpr uint32_t kTmAP = 0;     // + s * 64 (two A/P accumulators)
    static constexpr uint32_t kTmW = 128, kTmCols = 256;
};

struct KsParams {
    const __nv_bfloat16 *beta;
    const int32_t *cu;
    const int32_t *chunk_off;
    unsigned char *packets;
    long long slots;          // packets the workspace holds
    int32_t *status;
    int N, H;
};

__global__ void __launch_bounds__(kKsThreads, 1)
kside_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
             const __grid_constant__ CUtensorMap tm_la, KsParams p) {
    using Ly = KsLayout;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(sm);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + Ly::kBar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + Ly::kMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + Ly::kMisc + 4);
    float *sL = reinterpret_cast<float *>(sm + Ly::kL);
    float *sT = reinterpret_cast<float *>(sm + Ly::kT);
    float *sXw = reinterpret_cast<float *>(sm + Ly::kXw);
    float *sGP = reinterpret_cast<float *>(sm + Ly::kGP);
    float *sSUF = reinterpret_cast<float *>(sm + Ly::kSUF);
    float *sGL = reinterpret_cast<float *>(sm + Ly::kGL);
    float *sB = reinterpret_cast<float *>(sm + Ly::kB);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    long long total = (long long)p.chunk_off[p.N] * p.H;
    if (total > p.slots) {   // overlapping (malformed) sequences: never write past the workspace
        if (blockIdx.x == 0 && threadIdx.x == 0) set_status(p.status, KDA_ERR_SEQLENS);
        total = p.slots;
    }
    const long long first = blockIdx.x, stride = gridDim.x;
    const int count = first < total ? (int)((total - first + stride - 1) / stride) : 0;
    if (count == 0) return;

    if (tid == 0) {
        for (int i = 0; i < kbNum; ++i) {
            uint32_t cnt = 1;
            if (i == kbKqFull || i == kbKqFull + 1) cnt = kPrepThreads / 32;
            if (i == kbWReady || i == kbWReady + 1) cnt = 2;
            mbar_init(&bars[i], cnt);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kKsTma && lane == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_la);
    }
    for (int i = tid; i < 2 * 512; i += kKsThreads) {   // zero rows of both Tb|0|P tiles
        const int s = i / 512, j = i % 512;
        sts128(sbase + Ly::kTP + s * 24576 + 8192 + j * 16, 0, 0, 0, 0);
    }
    for (int i = tid; i < 64 * kLDL / 4; i += kKsThreads)  // T stays zero above its blocks
        sts128(sbase + Ly::kT + i * 16, 0, 0, 0, 0);
    if (warp == kKsMma) {
        tmem_alloc(tmem_slot, Ly::kTmCols);
        tmem_relinquish();
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == kKsTma) {
        // ------------------------------------------------------ TMA loads
        if (lane == 0) {
            for (int i = 0; i < count; ++i) {
                const int s = i & 1;
                // the packet of item i-2 must have left stage s
                if (i >= 2 && !wait_or_abort(&bars[kbStored + s], ((i - 2) >> 1) & 1, abort_flag,
                                             p.status))
                    break;
                const Item it = item_of(first + (long long)i * stride, p.H, p.chunk_off, p.cu, p.N);
                uint64_t *full = &bars[kbRawFull + s];
                mbar_arrive_expect_tx(full, 6 * 8192);
                for (int a = 0; a < 2; ++a) {
                    tma_load_3d(sm + Ly::kKQ + s * 32768 + a * 16384, &tm_k, full, a * 64, it.h, it.c0);
                    tma_load_3d(sm + Ly::kKQ + s * 32768 + a * 16384 + 8192, &tm_q, full, a * 64, it.h,
                                it.c0);
                    tma_load_3d(sm + Ly::kKI + s * 16384 + a * 8192, &tm_la, full, a * 64, it.h, it.c0);
                }
                KDA_TRACE1(i, 0);
                if (i + 2 < count) {   // warm L2 with the tiles this stage takes next
                    const Item nx = item_of(first + (long long)(i + 2) * stride, p.H, p.chunk_off,
                                            p.cu, p.N);
                    for (int a = 0; a < 2; ++a) {
                        tma_prefetch_3d(&tm_k, a * 64, nx.h, nx.c0);
                        tma_prefetch_3d(&tm_q, a * 64, nx.h, nx.c0);
                        tma_prefetch_3d(&tm_la, a * 64, nx.h, nx.c0);
                    }
                }
            }
            // armed loads must land before the CTA may exit
            for (int i = max(0, count - 2); i < count; ++i)
                mbar_wait(&bars[kbRawFull + (i & 1)], (i >> 1) & 1);
        }
    } else if (warp == kKsStore) {
        // ------------------------------------------------- packet stores
        // Each part of a packet leaves as soon as it is final: Qg, Ki and
        // Gam_L after the prep, Tb and P after the solve, -W last.
        if (lane == 0) {
            for (int i = 0; i < count; ++i) {
                const int s = i & 1;
                unsigned char *dst = p.packets + (size_t)(first + (long long)i * stride) * kPacketBytes;
                unsigned char *kq = sm + Ly::kKQ + s * 32768;
                unsigned char *tp = sm + Ly::kTP + s * 24576;
                if (!wait_or_abort(&bars[kbKqFull + s], (i >> 1) & 1, abort_flag, p.status)) break;
                bulk_store(dst + kPkKQ + 8192, kq + 8192, 8192);            // Qg, K atom 0
                bulk_store(dst + kPkKQ + 16384 + 8192, kq + 16384 + 8192, 8192);  // Qg, atom 1
                bulk_store(dst + kPkKI, sm + Ly::kKI + s * 16384, 16384);
                bulk_store(dst + kPkGL, sGL + s * 128, 512);
                bulk_commit();
                if (!wait_or_abort(&bars[kbTbFull + s], (i >> 1) & 1, abort_flag, p.status)) break;
                bulk_store(dst + kPkTb, tp, 8192);
                bulk_store(dst + kPkP, tp + 16384, 8192);
                bulk_commit();
                if (!wait_or_abort(&bars[kbWReady + s], (i >> 1) & 1, abort_flag, p.status)) break;
                bulk_store(dst + kPkKQ, kq, 8192);                           // -W, atom 0
                bulk_store(dst + kPkKQ + 16384, kq + 16384, 8192);           // -W, atom 1
                bulk_commit();
                KDA_TRACE1(i, 9);
                bulk_wait_read_all();
                KDA_TRACE1(i, 10);
                mbar_arrive(&bars[kbStored + s]);
            }
            bulk_wait_all();
        }
    } else if (warp >= kKsPrep0 && warp < kKsPrep0 + kPrepThreads / 32) {
        // ----------------------------------------------------------- prep
        const int t = tid - kKsPrep0 * 32;
        for (int i = 0; i < count; ++i) {
            const int s = i & 1;
            if (!wait_or_abort(&bars[kbRawFull + s], (i >> 1) & 1, abort_flag, p.status)) break;
            const Item it = item_of(first + (long long)i * stride, p.H, p.chunk_off, p.cu, p.N);
            if (t == 0) KDA_TRACE1(i, 1);
            prep_chunk(t, sbase + Ly::kKQ + s * 32768, sbase + Ly::kKI + s * 16384, sGP, sSUF,
                       sGL + s * 128, sB + s * 64, p.beta, it.c0, it.L, p.H, it.h, 1);
            if (t == 0) KDA_TRACE1(i, 2);
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[kbKqFull + s]);
        }
    } else if (warp >= kKsSolve0 && warp < kKsSolve0 + 4) {
        // ---------------------------------------------------------- solve
        const int sw = warp - kKsSolve0;
        const int t = tid - kKsSolve0 * 32;
        for (int i = 0; i < count; ++i) {
            const int s = i & 1;
            if (!wait_or_abort(&bars[kbApFull + s], (i >> 1) & 1, abort_flag, p.status)) break;
            tc_fence_after();
            if (t == 0) KDA_TRACE1(i, 4);
            solve_chunk(sw, lane, tmem, Ly::kTmAP + s * 64, sbase + Ly::kTP + s * 24576, sL, sT,
                        sXw, sB + s * 64, &bars[kbApFree + s], 2);
            if (t == 0) mbar_arrive(&bars[kbTbFull + s]);
            if (t == 0) KDA_TRACE1(i, 5);
            if (sw < 2) {
                if (!wait_or_abort(&bars[kbWaccFull], i & 1, abort_flag, p.status)) break;
                tc_fence_after();
                if (t == 0) KDA_TRACE1(i, 7);
                convert_w(sw, lane, tmem, Ly::kTmW, sbase + Ly::kKQ + s * 32768);
                if (lane == 0) mbar_arrive(&bars[kbWReady + s]);
                if (t == 0) KDA_TRACE1(i, 8);
            }
        }
    } else if (warp == kKsMma) {
        // ------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t kIdAP = idesc_bf16(128, 64, 0, 0);
            constexpr uint32_t kIdW = idesc_bf16(128, 128, 0, 1);
            for (int i = 0; i < count; ++i) {
                const int s = i & 1;
                const uint32_t kq = sbase + Ly::kKQ + s * 32768;
                const uint64_t d_kq = smem_desc(kq, 16, 1024, kSw128);
                const uint64_t d_ki = smem_desc(sbase + Ly::kKI + s * 16384, 16, 1024, kSw128);
                const uint64_t d_tp = smem_desc(sbase + Ly::kTP + s * 24576, 16, 1024, kSw128);
                const uint64_t d_kg = smem_desc(kq, 16384, 1024, kSw128);
                if (!wait_or_abort(&bars[kbKqFull + s], (i >> 1) & 1, abort_flag, p.status)) break;
                if (i >= 2 && !wait_or_abort(&bars[kbApFree + s], ((i - 2) >> 1) & 1, abort_flag,
                                             p.status))
                    break;
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_bf16(tmem + Ly::kTmAP + s * 64, d_kq + kmaj_step(ks, 16384),
                             d_ki + kmaj_step(ks, 8192), kIdAP, ks > 0);
                mma_commit(&bars[kbApFull + s]);
                KDA_TRACE1(i, 3);
                if (!wait_or_abort(&bars[kbTbFull + s], (i >> 1) & 1, abort_flag, p.status)) break;
                if (i >= 1 && !wait_or_abort(&bars[kbWReady + ((i - 1) & 1)], ((i - 1) >> 1) & 1,
                                             abort_flag, p.status))
                    break;
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tmem + Ly::kTmW, d_tp + ((uint64_t)(ks * 32) >> 4),
                             d_kg + ((uint64_t)(ks * 2048) >> 4), kIdW, ks > 0);
                mma_commit(&bars[kbWaccFull]);
                KDA_TRACE1(i, 6);
            }
            mma_commit(&bars[kbDrain]);
            mbar_wait(&bars[kbDrain], 0);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kKsMma) {
        tc_fence_after();
        tmem_dealloc(tmem, Ly::kTmCols);
    }
}

// ============================================================ pass 2
constexpr int kChWarps = 6;   // 0-3 chain, 4 loader, 5 MMA
constexpr int kChThreads = kChWarps * 32;
enum ChRole { kChLoad = 4, kChMma = 5 };
enum ChBars {
    cbFull = 0,       // [2] packet + value tile landed
    cbStageFree = 2,  // [2] every MMA of a stage done
    cbSbFull = 4,     // count 4
    cbUFull = 5,
    cbUbFull = 6,     // count 2
    cbDsFull = 7,
    cbOFull = 8,      // [2]
    cbD1Free = 10,    // [2] count 2
    cbDrain = 12,
    cbNum = 13
};

template <int VS>
struct ChLayout {
    static constexpr uint32_t kKQ = 0, kKI = 32768, kTP = 49152, kV = 73728;
    static constexpr uint32_t kGL = kV + 64 * VS * 2;     // 512 B
    static constexpr uint32_t kStage = (kGL + 512 + 1023) / 1024 * 1024;  // KQ | KI | TP | V | GL
    static constexpr uint32_t kSB = 2 * kStage;
    static constexpr uint32_t kUB = kSB + 128 * VS * 2;
    static constexpr uint32_t kBar = kUB + 64 * VS * 2;
    static constexpr uint32_t kMisc = kBar + 16 * 8;
    static constexpr uint32_t kAlloc = kMisc + 16 + 1024;
    static_assert(kAlloc <= 232448, "shared memory budget exceeded");
    static constexpr uint32_t kTmD1 = 0;          // + s * VS
    static constexpr uint32_t kTmD2 = 2 * VS;
    static constexpr uint32_t kTmCols = 128;
};

struct ChParams {
    const float *S0;
    const int32_t *cu;
    const int32_t *chunk_off;
    const unsigned char *packets;
    long long slots;
    __nv_bfloat16 *out;
    float *Sf;
    const int32_t *order;
    int32_t *status;
    int N, T, H;
};

template <int VS>
__global__ void __launch_bounds__(kChThreads, 1)
chain_kernel(const __grid_constant__ CUtensorMap tm_v, ChParams p) {
    using Ly = ChLayout<VS>;
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
    if ((long long)(g0 + nchunks) * p.H > p.slots) {
        if (tid == 0) set_status(p.status, KDA_ERR_SEQLENS);
        return;
    }
    const size_t sbase_g = ((size_t)seq * p.H + h) * kDK * kDV + (size_t)vs * VS;

    if (tid == 0) {
        for (int i = 0; i < cbNum; ++i) {
            uint32_t cnt = 1;
            if (i == cbSbFull) cnt = 4;
            if (i == cbUbFull) cnt = 2;
            if (i == cbD1Free || i == cbD1Free + 1) cnt = 2;
            mbar_init(&bars[i], cnt);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kChLoad && lane == 0) prefetch_tmap(&tm_v);
    for (int i = tid; i < 2 * 512; i += kChThreads) {   // zero rows of both Tb|0|P tiles
        const int s = i / 512, j = i % 512;
        sts128(sbase + s * Ly::kStage + Ly::kTP + 8192 + j * 16, 0, 0, 0, 0);
    }
    if (warp == kChMma) {
        tmem_alloc(tmem_slot, Ly::kTmCols);
        tmem_relinquish();
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    auto packet = [&](int j) {
        return p.packets + ((size_t)(g0 + j) * p.H + h) * kPacketBytes;
    };

    if (warp == kChLoad) {
        // ------------------------------------------------------- loader
        if (lane == 0) {
            for (int j = 0; j < nchunks; ++j) {
                const int s = j & 1;
                if (j >= 2 && !wait_or_abort(&bars[cbStageFree + s], ((j - 2) >> 1) & 1, abort_flag,
                                             p.status))
                    break;
                unsigned char *st = sm + s * Ly::kStage;
                const unsigned char *src = packet(j);
                uint64_t *full = &bars[cbFull + s];
                mbar_arrive_expect_tx(full, 65536 + 512 + 64 * VS * 2);
                bulk_load(st + Ly::kKQ, src + kPkKQ, 32768, full);
                bulk_load(st + Ly::kKI, src + kPkKI, 16384, full);
                bulk_load(st + Ly::kTP, src + kPkTb, 8192, full);
                bulk_load(st + Ly::kTP + 16384, src + kPkP, 8192, full);
                bulk_load(st + Ly::kGL, src + kPkGL, 512, full);
                tma_load_3d(st + Ly::kV, &tm_v, full, vs * VS, h, t0 + j * kChunk);
                KDA_TRACE2(j, 0);
                if (j + 2 < nchunks) bulk_prefetch_l2(packet(j + 2), kPkGL + 512);
            }
            for (int j = max(0, nchunks - 2); j < nchunks; ++j)
                mbar_wait(&bars[cbFull + (j & 1)], (j >> 1) & 1);
        }
    } else if (warp == kChMma) {
        // ------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t kIdV = idesc_bf16(128, VS, 0, 1);
            constexpr uint32_t kIdS = idesc_bf16(128, VS, 1, 1);
            const uint64_t d_sb = vs_desc<VS>(sbase + Ly::kSB, 128);
            const uint64_t d_ub = vs_desc<VS>(sbase + Ly::kUB, 64);
            for (int j = 0; j < nchunks; ++j) {
                const int s = j & 1;
                const uint32_t st = sbase + s * Ly::kStage;
                const uint32_t d1 = tmem + Ly::kTmD1 + s * VS;
                const uint64_t d_kq = smem_desc(st + Ly::kKQ, 16, 1024, kSw128);
                const uint64_t d_kit = smem_desc(st + Ly::kKI, 8192, 1024, kSw128);
                const uint64_t d_tp = smem_desc(st + Ly::kTP, 16, 1024, kSw128);
                const uint64_t d_p = smem_desc(st + Ly::kTP + 8192, 16, 1024, kSw128);
                const uint64_t d_v = vs_desc<VS>(st + Ly::kV, 64);
                if (!wait_or_abort(&bars[cbFull + s], (j >> 1) & 1, abort_flag, p.status)) break;
                if (j >= 2 && !wait_or_abort(&bars[cbD1Free + s], ((j - 2) >> 1) & 1, abort_flag,
                                             p.status))
                    break;
                KDA_TRACE2(j, 1);
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)   // D1 = Tb V (U0; zero in rows 64..127)
                    mma_bf16(d1, d_tp + ((uint64_t)(ks * 32) >> 4), d_v + vs_step<VS>(ks), kIdV,
                             ks > 0);
                if (!wait_or_abort(&bars[cbSbFull], j & 1, abort_flag, p.status)) break;
                KDA_TRACE2(j, 2);
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)   // D1 += [-W; Qg] S
                    mma_bf16(d1, d_kq + kmaj_step(ks, 16384), d_sb + vs_step<VS>(ks), kIdV, 1);
                mma_commit(&bars[cbUFull]);
                KDA_TRACE2(j, 3);
                if (!wait_or_abort(&bars[cbUbFull], j & 1, abort_flag, p.status)) break;
                KDA_TRACE2(j, 4);
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)   // dS = Ki^T U
                    mma_bf16(tmem + Ly::kTmD2, d_kit + ((uint64_t)(ks * 2048) >> 4),
                             d_ub + vs_step<VS>(ks), kIdS, ks > 0);
                mma_commit(&bars[cbDsFull]);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)   // D1 += [0; P] U  (O)
                    mma_bf16(d1, d_p + ((uint64_t)(ks * 32) >> 4), d_ub + vs_step<VS>(ks), kIdV, 1);
                mma_commit(&bars[cbOFull + s]);
                mma_commit(&bars[cbStageFree + s]);
                KDA_TRACE2(j, 5);
            }
            mma_commit(&bars[cbDrain]);
            mbar_wait(&bars[cbDrain], 0);
        }
    } else {
        // ------------------------------------------------------ chain warps
        const int c = tid;                 // state row (key channel) 0..127
        const int wq = warp;               // TMEM lane quarter
        float S[VS];
        {
            const float *src = p.S0 ? p.S0 + sbase_g + (size_t)c * kDV : nullptr;
#pragma unroll
            for (int jj = 0; jj < VS; jj += 4) {
                float4 v = src ? *reinterpret_cast<const float4 *>(src + jj) : make_float4(0, 0, 0, 0);
                S[jj] = v.x; S[jj + 1] = v.y; S[jj + 2] = v.z; S[jj + 3] = v.w;
            }
        }
        auto store_out = [&](int m) {
            const int sm1 = m & 1;
            const int c0 = t0 + m * kChunk, L = min(kChunk, t1 - c0);
            const int r = c - 64;
#pragma unroll
            for (int jj = 0; jj < VS; jj += 32) {
                uint32_t v[32];
                tmem_ld32(tmem_addr(tmem, 32 * wq, Ly::kTmD1 + sm1 * VS + jj), v);
                tmem_wait_ld();
                if (r < L) {
                    __nv_bfloat16 *dst = p.out + ((size_t)(c0 + r) * p.H + h) * kDV + vs * VS + jj;
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
        for (int j = 0; j <= nchunks && ok; ++j) {
            if (j > 0) {
                // S <- Diag(Gam_L) (S + dS) for chunk j-1
                if (!wait_or_abort(&bars[cbDsFull], (j - 1) & 1, abort_flag, p.status)) { ok = false; break; }
                tc_fence_after();
                if (c == 0) KDA_TRACE2(j - 1, 6);
#pragma unroll
                for (int jj = 0; jj < VS; jj += 32) {
                    uint32_t v[32];
                    tmem_ld32(tmem_addr(tmem, 32 * wq, Ly::kTmD2 + jj), v);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) S[jj + e] = gl_cur * (S[jj + e] + __uint_as_float(v[e]));
                }
            }
            if (j == nchunks) {
                if (wq >= 2 && j > 0) {
                    const int m = j - 1;
                    if (!wait_or_abort(&bars[cbOFull + (m & 1)], (m >> 1) & 1, abort_flag, p.status)) { ok = false; break; }
                    tc_fence_after();
                    store_out(m);
                }
                break;
            }
            const int s = j & 1;
            if (!wait_or_abort(&bars[cbFull + s], (j >> 1) & 1, abort_flag, p.status)) { ok = false; break; }
            gl_cur = reinterpret_cast<const float *>(sm + s * Ly::kStage + Ly::kGL)[c];
            if (c == 0) KDA_TRACE2(j, 7);
            {
                const uint32_t sb = sbase + Ly::kSB;
#pragma unroll
                for (int q8 = 0; q8 < VS / 8; ++q8) {
                    sts128(sb + vs_off<VS>(c, q8), pack2(S[8 * q8], S[8 * q8 + 1]),
                           pack2(S[8 * q8 + 2], S[8 * q8 + 3]), pack2(S[8 * q8 + 4], S[8 * q8 + 5]),
                           pack2(S[8 * q8 + 6], S[8 * q8 + 7]));
                }
            }
            fence_proxy_async();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[cbSbFull]);
            if (c == 0) KDA_TRACE2(j, 8);

            if (wq < 2) {
                // U rows: D1 lanes 0..63 -> bf16 operand
                if (!wait_or_abort(&bars[cbUFull], j & 1, abort_flag, p.status)) { ok = false; break; }
                tc_fence_after();
                if (c == 0) KDA_TRACE2(j, 9);
                const uint32_t ub = sbase + Ly::kUB;
#pragma unroll
                for (int jj = 0; jj < VS; jj += 32) {
                    uint32_t v[32];
                    tmem_ld32(tmem_addr(tmem, 32 * wq, Ly::kTmD1 + s * VS + jj), v);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; e += 8) {
                        sts128(ub + vs_off<VS>(c, (jj + e) / 8),
                               pack2(__uint_as_float(v[e]), __uint_as_float(v[e + 1])),
                               pack2(__uint_as_float(v[e + 2]), __uint_as_float(v[e + 3])),
                               pack2(__uint_as_float(v[e + 4]), __uint_as_float(v[e + 5])),
                               pack2(__uint_as_float(v[e + 6]), __uint_as_float(v[e + 7])));
                    }
                }
                fence_proxy_async();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[cbUbFull]);
                if (c == 0) KDA_TRACE2(j, 10);
            } else if (j > 0) {
                const int m = j - 1;
                if (!wait_or_abort(&bars[cbOFull + (m & 1)], (m >> 1) & 1, abort_flag, p.status)) { ok = false; break; }
                tc_fence_after();
                store_out(m);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[cbD1Free + (m & 1)]);
            }
        }
        if (ok && p.Sf) {
            float *dst = p.Sf + sbase_g + (size_t)c * kDV;
#pragma unroll
            for (int jj = 0; jj < VS; jj += 4)
                *reinterpret_cast<float4 *>(dst + jj) = make_float4(S[jj], S[jj + 1], S[jj + 2], S[jj + 3]);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kChMma) {
        tc_fence_after();
        tmem_dealloc(tmem, Ly::kTmCols);
    }
}

int sm_count() {
    static int n = 0;
    if (!n) {
        int dev = 0;
        cudaGetDevice(&dev);
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
    }
    return n;
}

}  // namespace

cudaError_t launch_prefill_two_pass(const ForwardArgs &a, cudaStream_t s) {
    constexpr int VS = 32;
    const int T = a.T > 0 ? a.T : 1;
    CUtensorMap mq, mk, mla, mv;
    if (!make_tmap_bf16_3d(&mq, a.q, T, a.H, kDK, 64, 128) ||
        !make_tmap_bf16_3d(&mk, a.k, T, a.H, kDK, 64, 128) ||
        !make_tmap_bf16_3d(&mla, a.log_alpha, T, a.H, kDK, 64, 128) ||
        !make_tmap_bf16_3d(&mv, a.v, T, a.H, kDV, VS, VS * 2))
        return cudaErrorInvalidValue;
    // pass 1: persistent, at most one CTA per SM, items strided over the grid
    KsParams kp;
    kp.beta = static_cast<const __nv_bfloat16 *>(a.beta);
    kp.cu = a.cu_seqlens;
    kp.chunk_off = a.chunk_off;
    kp.packets = a.packets;
    kp.slots = (long long)a.packet_slots;
    kp.status = a.status;
    kp.N = a.N;
    kp.H = a.H;
    cudaError_t e = cudaFuncSetAttribute(kside_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)KsLayout::kAlloc);
    if (e != cudaSuccess) return e;
    const size_t items = a.packet_slots;
    const unsigned grid1 = (unsigned)(items < (size_t)sm_count() ? items : (size_t)sm_count());
    kside_kernel<<<grid1, kKsThreads, KsLayout::kAlloc, s>>>(mq, mk, mla, kp);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // pass 2: one CTA per (sequence, head, value slice), longest sequences first
    ChParams cp;
    cp.S0 = a.S0;
    cp.cu = a.cu_seqlens;
    cp.chunk_off = a.chunk_off;
    cp.packets = a.packets;
    cp.slots = (long long)a.packet_slots;
    cp.out = static_cast<__nv_bfloat16 *>(a.out);
    cp.Sf = a.S_final;
    cp.order = a.order;
    cp.status = a.status;
    cp.N = a.N;
    cp.T = a.T;
    cp.H = a.H;
    auto kern = chain_kernel<VS>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)ChLayout<VS>::kAlloc);
    if (e != cudaSuccess) return e;
    const unsigned grid2 = (unsigned)a.N * a.H * (kDV / VS);
    kern<<<grid2, kChThreads, ChLayout<VS>::kAlloc, s>>>(mv, cp);
    return cudaGetLastError();
}

}  // namespace kda

#ifdef KDA_TRACE
extern "C" int kda_trace1_read(unsigned long long *host) {
    return (int)cudaMemcpyFromSymbol(host, kda::g_kda_trace1, sizeof(kda::g_kda_trace1));
}
extern "C" int kda_trace2_read(unsigned long long *host) {
    return (int)cudaMemcpyFromSymbol(host, kda::g_kda_trace2, sizeof(kda::g_kda_trace2));
}
#endif
