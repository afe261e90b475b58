// kda_prefill_2pass.cu -- two-pass tensor-core KDA prefill (bf16 I/O, fp32 state).
//
// The chunked evaluation of the recurrence of the page "Kimi K3: Open Frontier
// Intelligence and Implementation Framework" (section "Hybrid Attention
// Mechanism", KDA bullet) splits into work that depends only on one chunk's
// keys, queries and gates, and a short sequential state chain.  The key-side
// work dominates the latency of a chunk, so it runs in its own pass:
//
//   pass 1  (kside_kernel, persistent, one chunk x head per item, spread over
//           every SM, items claimed from a counter): gate prep, [A;P] =
//           [Kg;Qg] Ki^T, the triangular inverse Tb, PT = P Tb and
//           [W; PW] = [Tb; PT] Kg.  It writes one operand packet per item to
//           the workspace, in the exact shared-memory layout pass 2 consumes:
//             [-W;Qe] 32 KB | Ki 16 KB | [Tb;PT] 16 KB | Gam_L 512 B
//           with Qe = Qg - P W.
//   pass 2  (chain_kernel, one CTA per (sequence, head, VS-wide value slice)):
//           streams the packets and the value tile with bulk copies and runs
//           only the value-side products and the fp32 state chain:
//             D1  = [Tb;PT] V ; D1 += [-W;Qe] S   (rows: U | O = Qg S + P U)
//             dS  = Ki^T U ;  S <- Diag(Gam_L) (S + dS)
//
// The packets cost ~1 KB of extra HBM traffic per token-head each way
// (written once, read once; the value slices of a chain share each packet
// through L2).  Pass 1 and pass 2 are launched as programmatic dependents of
// the kernel before them.
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
// per-CTA [globaltimer start, end, clock64 start, end] of both passes
__device__ unsigned long long g_kda_span1[1024 * 4];
__device__ unsigned long long g_kda_span2[1024 * 4];
#define KDA_SPAN(buf, k)                                                                   \
    do {                                                                                   \
        if (threadIdx.x == 0 && blockIdx.x < 1024) {                                       \
            buf[blockIdx.x * 4 + (k)] = globaltimer_ns();                                  \
            buf[blockIdx.x * 4 + 2 + (k)] = clock64();                                     \
        }                                                                                  \
    } while (0)
#else
#define KDA_SPAN(buf, k) \
    do {                 \
    } while (0)
#define KDA_TRACE1(n, e) \
    do {                 \
    } while (0)
#define KDA_TRACE2(n, e) \
    do {                 \
    } while (0)
#endif

// Packet layout (bytes).  Every tile is the 128-byte-swizzled K-major image
// the chain pass hands to the tensor cores as it lands:
//   [-W; Qe]  two 16 KB atoms (channels 0-63, 64-127) of 128 rows: rows
//             0-63 = -W = -Tb Kg, rows 64-127 = Qe = Qg - P W
//   Ki        two 8 KB atoms of 64 rows
//   [Tb; PT]  128 rows x 64 positions: Tb = T diag(b), PT = P Tb
//   Gam_L     128 fp32 channel decays of the whole chunk
// With these the chain computes U = Tb V - W S and O = Qe S + PT V, which
// equals Qg S + P U: the intra-chunk output needs no product after U.
constexpr uint32_t kPkKQ = 0;
constexpr uint32_t kPkKI = 32768;
constexpr uint32_t kPkTP = 49152;
constexpr uint32_t kPkGL = 65536;
static_assert(kPkGL + 512 <= kPacketBytes, "packet layout");

// PT = P Tb into bf16 rows 64..127 of the Tb|PT tile, on the four solve
// warps with the warp-level bf16 MMA (fp32 accumulation, as a tcgen05
// product would): warp sw owns columns 16 sw .. 16 sw + 15 of every row; P is
// lower-inclusive, so row tile mt sums key tiles 0..mt only.  Doing this here
// saves a tensor-memory round trip between the solve and the W product.
__device__ __forceinline__ void pt_product(int sw, int lane, uint32_t p_tile, uint32_t tp) {
    const int l7 = lane & 7, mi = lane >> 3, g = lane >> 2, tq = lane & 3;
    // B fragments of this warp's two column tiles for the four key tiles,
    // loaded once; ten independent accumulator chains of at most 4 products
    uint32_t bf[4][4];
#pragma unroll
    for (int ks = 0; ks < 4; ++ks)
        ldsm_x4_t(tp + sw128_off(16 * ks + l7 + (mi & 1) * 8, 2 * sw + (mi >> 1)), bf[ks]);
    float acc[4][2][4];
#pragma unroll
    for (int mt = 0; mt < 4; ++mt)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[mt][nt][e] = 0.f;
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
#pragma unroll
        for (int mt = ks; mt < 4; ++mt) {
            uint32_t af[4];
            ldsm_x4(p_tile + sw128_off(16 * mt + l7 + (mi & 1) * 8, 2 * ks + (mi >> 1)), af);
            mma16816(acc[mt][0], af, bf[ks][0], bf[ks][1]);
            mma16816(acc[mt][1], af, bf[ks][2], bf[ks][3]);
        }
    }
#pragma unroll
    for (int mt = 0; mt < 4; ++mt)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const int r = 64 + 16 * mt + g, chunk = 2 * sw + nt;
            sts32(tp + sw128_off(r, chunk) + 4 * tq, pack2(acc[mt][nt][0], acc[mt][nt][1]));
            sts32(tp + sw128_off(r + 8, chunk) + 4 * tq, pack2(acc[mt][nt][2], acc[mt][nt][3]));
        }
}

// [W; PW] (TMEM lanes 0..127) -> -W over the Kg rows and Qe = Qg - PW over
// the Qg rows of the key-query tile, as bf16.  Run by the eight prep warps:
// warp w owns rows 32 (w % 4) .. + 31 and the 64 channels of atom w / 4.
__device__ __forceinline__ void convert_wqe8(int w, int lane, uint32_t tmem, uint32_t tm_w,
                                             uint32_t kq_stage) {
    const int qt = w & 3, hh = w >> 2;
    const int r = 32 * qt + lane;
    // one code path for both halves: -W = 0 - W over the Kg rows, Qe = Qg - PW
    const uint32_t keep = qt < 2 ? 0u : 0xFFFFFFFFu;
#pragma unroll 1
    for (int half = 0; half < 2; ++half) {
        uint32_t v[32];
        tmem_ld32(tmem_addr(tmem, 32 * qt, tm_w + 64 * hh + 32 * half), v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t addr = kq_stage + hh * 16384 + sw128_off(r, 4 * half + j);
            const uint4 qv = lds128(addr);
            const uint32_t qw[4] = {qv.x & keep, qv.y & keep, qv.z & keep, qv.w & keep};
            uint32_t o[4];
#pragma unroll
            for (int e2 = 0; e2 < 4; ++e2)
                o[e2] = pack2(bf16lo(qw[e2]) - __uint_as_float(v[8 * j + 2 * e2]),
                              bf16hi(qw[e2]) - __uint_as_float(v[8 * j + 2 * e2 + 1]));
            sts128(addr, o[0], o[1], o[2], o[3]);
        }
    }
    fence_proxy_async();
    tc_fence_before();
    __syncwarp();
}

// ============================================================ pass 1
constexpr int kKsWarps = 15;   // 0-7 prep, 8-11 solve, 12 TMA loads, 13 MMA, 14 packet stores
constexpr int kKsThreads = kKsWarps * 32;
enum KsRole { kKsPrep0 = 0, kKsSolve0 = 8, kKsTma = 12, kKsMma = 13, kKsStore = 14 };
// Item i holds key-query stage i % kKqStages from its load until its packet
// has left (most of the pipeline) and gate stage i % kKiStages only until the
// A/P product and the Ki store have read it, so the key-query ring is deeper.
constexpr int kKqStages = 4;   // raw k|q -> Kg|Qg -> -W|Qe
constexpr int kKiStages = 2;   // raw log_alpha -> prefix scratch -> Ki
enum KsBars {
    kbRawFull = 0,   // [4] TMA -> prep (per key-query stage; covers the gate tiles)
    kbKqFull = 4,    // [4] count 8: prep -> A/P issuer, Ki stores
    kbApFull = 8,    // [2] A/P product -> solve (two TMEM accumulators)
    kbApFree = 10,   // [2] solve has read D_AP[s] -> A/P issuer
    kbTbFull = 12,   // solve -> W issuer (Tb and PT written)
    kbTpFree = 13,   // the Tb|PT tile has been read -> Tb write of the next chunk
    kbWaccFull = 14, // [W; PW] product -> prep warps
    kbWReady = 15,   // count 8: -W and Qe written -> stores (and D_W free)
    kbStored = 16,   // [4] the packet's -W|Qe copies have read the key-query stage -> TMA
    kbKiFree = 20,   // [2] count 4: A/P product done, Ki and Gam_L copies read -> TMA
    kbDrain = 22,    // [2] A/P issuer, W issuer
    kbNum = 24
};

struct KsLayout {
    static constexpr uint32_t kKQ = 0;                              // 4 x 32 KB
    static constexpr uint32_t kKI = kKQ + kKqStages * 32768;        // 2 x 16 KB (also the prep's scan scratch)
    static constexpr uint32_t kTP = kKI + kKiStages * 16384;        // 16 KB: Tb | PT
    static constexpr uint32_t kP = kTP + 16384;                       // 8 KB: P
    static constexpr uint32_t kL = kP + 8192;
    static constexpr uint32_t kT = kL + 64 * kLDL * 4;
    static constexpr uint32_t kGL = kT + 64 * kLDL * 4;     // [2][128], per gate stage
    static constexpr uint32_t kB = kGL + kKiStages * 128 * 4;       // [4][64], per key-query stage
    static constexpr uint32_t kBar = kB + kKqStages * 64 * 4;
    static constexpr uint32_t kMisc = kBar + kbNum * 8;
    static constexpr uint32_t kItem = kMisc + 16;   // [4] Item of each key-query stage
    static constexpr uint32_t kAlloc = kItem + kKqStages * sizeof(Item) + 1024;
    static_assert(kAlloc <= 232448, "shared memory budget exceeded");
    static constexpr uint32_t kTmAP = 0;     // + (i & 1) * 64 (two A/P accumulators)
    static constexpr uint32_t kTmW = 128;    // [W; PW], 128 columns
    static constexpr uint32_t kTmCols = 256;
};

struct KsParams {
    const __nv_bfloat16 *beta;
    const int32_t *cu;
    const int32_t *chunk_off;
    unsigned char *packets;
    long long slots;          // packets the workspace holds
    int32_t *status;
    int32_t *work_ctr;        // items past the first wave are claimed from here
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
    float *sGL = reinterpret_cast<float *>(sm + Ly::kGL);
    float *sB = reinterpret_cast<float *>(sm + Ly::kB);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // Launched as a programmatic dependent of the varlen index: the chain
    // pass may be scheduled onto SMs as this pass's CTAs finish, and the
    // chunk offsets and item counter are read only after the index is done.
    grid_launch_dependents();
    grid_dependency_wait();
    long long total = (long long)p.chunk_off[p.N] * p.H;
    if (total < 0 || total > p.slots) {   // overlapping (malformed) sequences: never write past the workspace
        if (blockIdx.x == 0 && threadIdx.x == 0) set_status(p.status, KDA_ERR_SEQLENS);
        total = p.slots;
    }
    // Each CTA starts on item blockIdx.x and claims further items from a
    // counter as its loader frees a stage, so CTAs that run faster (SMs vary
    // by several percent here) take more of the work.
    if ((long long)blockIdx.x >= total) return;
    Item *items = reinterpret_cast<Item *>(sm + Ly::kItem);

    if (tid == 0) {
        for (int i = 0; i < kbNum; ++i) {
            uint32_t cnt = 1;
            if (i >= kbKqFull && i < kbKqFull + kKqStages) cnt = kPrepThreads / 32;
            if (i == kbWReady) cnt = kPrepThreads / 32;
            if (i >= kbKiFree && i < kbKiFree + kKiStages) cnt = 4;
            mbar_init(&bars[i], cnt);
        }
        abort_flag[0] = 0;
        abort_flag[1] = 0;
        fence_mbar_init();
    }
    if (warp == kKsTma && lane == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_la);
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
    KDA_SPAN(g_kda_span1, 0);

    if (warp == kKsTma) {
        // ------------------------------------------------------ TMA loads
        // Copies issued by one thread are serviced one after another, so each
        // of the six tiles of a stage is issued by its own lane.
        // Items are claimed three ahead of their load so their tiles can be
        // warmed in L2; lane 0 claims and looks the coordinates up (global
        // memory) and broadcasts them.
        bool claimed_out = false;
        auto claim = [&](bool first_item) -> Item {
            Item it;
            it.h = it.c0 = it.L = 0;
            it.m = -1;
            if (lane == 0 && !claimed_out) {
                const long long m = first_item ? (long long)blockIdx.x
                                               : (long long)gridDim.x + atomicAdd(p.work_ctr, 1);
                if (m < total) it = item_of(m, p.H, p.chunk_off, p.cu, p.N);
            }
            it.h = __shfl_sync(0xffffffffu, it.h, 0);
            it.c0 = __shfl_sync(0xffffffffu, it.c0, 0);
            it.L = __shfl_sync(0xffffffffu, it.L, 0);
            it.m = __shfl_sync(0xffffffffu, it.m, 0);
            if (it.m < 0) claimed_out = true;
            return it;
        };
        const int a = lane & 1, which = lane >> 1;   // lanes 0-5: atom a of k, q or log_alpha
        const CUtensorMap *tm = which == 0 ? &tm_k : which == 1 ? &tm_q : &tm_la;
        auto warm = [&](const Item &it) {   // L2 prefetch of an item's tiles
            if (it.m >= 0 && lane < 6) tma_prefetch_3d(tm, a * 64, it.h, it.c0);
        };
        // nx0..nx2: the next three items; iterations -3..-1 only fill them,
        // so claim() and warm() have one call site each
        Item nx0, nx1, nx2;
        nx0.m = nx1.m = nx2.m = -1;
        nx0.h = nx1.h = nx2.h = nx0.c0 = nx1.c0 = nx2.c0 = nx0.L = nx1.L = nx2.L = 0;
        int n_loaded = 0;
        bool ended = false;
#pragma unroll 1
        for (int i = -3;; ++i) {
            if (i >= 0) {
                const int s = i % kKqStages, si = i % kKiStages;
                const Item it = nx0;
                // the packet of item i-4 must have left key-query stage s
                bool ok = true;
                if (lane == 0 && i >= kKqStages)
                    ok = wait_or_abort(&bars[kbStored + s], ((i / kKqStages) - 1) & 1, abort_flag,
                                       p.status);
                // and item i-2 must be done with gate stage si
                if (lane == 0 && ok && it.m >= 0 && i >= kKiStages)
                    ok = wait_or_abort(&bars[kbKiFree + si], ((i / kKiStages) - 1) & 1, abort_flag,
                                       p.status);
                if (!__shfl_sync(0xffffffffu, ok, 0)) break;
                uint64_t *full = &bars[kbRawFull + s];
                if (it.m < 0) {   // no more items: tell the prep, which tells the rest
                    if (lane == 0) {
                        items[s] = it;
                        mbar_arrive(full);
                    }
                    ended = true;
                    break;
                }
                if (lane == 0) {
                    items[s] = it;
                    mbar_arrive_expect_tx(full, 6 * 8192);
                }
                __syncwarp();
                if (lane < 6) {
                    const uint32_t dst = which < 2 ? Ly::kKQ + s * 32768 + a * 16384 + which * 8192
                                                   : Ly::kKI + si * 16384 + a * 8192;
                    tma_load_3d(sm + dst, tm, full, a * 64, it.h, it.c0);
                }
                if (lane == 0) KDA_TRACE1(i, 0);
                n_loaded = i + 1;
            }
            nx0 = nx1;
            nx1 = nx2;
            nx2 = claim(i == -3);
            if (i > -3) warm(nx2);
        }
        // Armed loads must land before the CTA may exit.  The end marker went
        // to the stage of item n_loaded - 4, whose load the Stored wait above
        // already saw consumed (and whose phase the marker has moved past).
        if (lane == 0)
            for (int i = max(0, n_loaded - kKqStages + (ended ? 1 : 0)); i < n_loaded; ++i)
                mbar_wait(&bars[kbRawFull + i % kKqStages], (i / kKqStages) & 1);
    } else if (warp == kKsStore) {
        // ------------------------------------------------- packet stores
        // Lane 0 waits and issues the products that follow the solve; the
        // copies are spread over lanes, each lane tracking its own groups.
#pragma unroll 1
        for (int i = 0;; ++i) {
            const int s = i % kKqStages;
            unsigned char *kq = sm + Ly::kKQ + s * 32768;
            unsigned char *tp = sm + Ly::kTP;
            bool ok = true;
            // The W product is issued here rather than by the A/P issuer, so
            // the next chunk's A/P product never queues behind this chunk's
            // solve.  D_W is free: this lane already waited for the previous
            // chunk's conversion out of it.
            if (lane == 0) ok = wait_or_abort(&bars[kbTbFull], i & 1, abort_flag, p.status);
            if (!__shfl_sync(0xffffffffu, ok, 0)) break;
            const int m = items[s].m;
            if (m < 0) break;
            if (!KDA_IN_RANGE((long long)m < p.slots, p.status)) break;
            unsigned char *dst = p.packets + (size_t)m * kPacketBytes;
            if (lane == 0) {   // [W; PW] = [Tb; PT] Kg
                tc_fence_after();
                constexpr uint32_t kIdW = idesc_bf16(128, 128, 0, 1);
                const uint64_t d_tp = smem_desc(sbase + Ly::kTP, 16, 1024, kSw128);
                const uint64_t d_kg = smem_desc(smem_u32(kq), 16384, 1024, kSw128);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tmem + Ly::kTmW, d_tp + ((uint64_t)(ks * 32) >> 4),
                             d_kg + ((uint64_t)(ks * 2048) >> 4), kIdW, ks > 0);
                mma_commit(&bars[kbWaccFull]);
                KDA_TRACE1(i, 6);
                bulk_store(dst + kPkTP, tp, 16384);
                bulk_commit();
                bulk_wait_read_all();
                mma_commit(&bars[kbTpFree]);   // after both products have read the tile
                ok = wait_or_abort(&bars[kbWReady], i & 1, abort_flag, p.status);
            }
            if (!__shfl_sync(0xffffffffu, ok, 0)) break;
            if (lane < 4) {   // [-W; Qe] in four 8 KB pieces, one per lane
                bulk_store(dst + kPkKQ + lane * 8192, kq + lane * 8192, 8192);
                bulk_commit();
            }
            if (lane == 0) KDA_TRACE1(i, 9);
            bulk_wait_read_all();
            __syncwarp();
            if (lane == 0) {
                KDA_TRACE1(i, 10);
                mbar_arrive(&bars[kbStored + s]);
            }
        }
        if (lane == 0) {
            mma_commit(&bars[kbDrain + 1]);   // every product of this lane done before TMEM is freed
            mbar_wait(&bars[kbDrain + 1], 0);
        }
        bulk_wait_all();
    } else if (warp >= kKsPrep0 && warp < kKsPrep0 + kPrepThreads / 32) {
        // ----------------------------------------------------------- prep
        const int t = tid - kKsPrep0 * 32;
        // After preparing chunk i these warps turn chunk i-2's [W; PW] product
        // into the bf16 -W and Qe operands.
        // Thread 0 waits on each mbarrier and named_bar_or() shares the
        // outcome: the eight warps leave together on a failed wait, so none is
        // left at one of prep_chunk's named barriers.
        auto convert = [&](int m) -> bool {
            const int sm4 = m % kKqStages;
            const bool w = t != 0 || wait_or_abort(&bars[kbWaccFull], m & 1, abort_flag, p.status);
            if (named_bar_or(1, kPrepThreads, !w)) return false;
            tc_fence_after();
            if (t == 0) KDA_TRACE1(m, 7);
            convert_wqe8(warp, lane, tmem, Ly::kTmW, sbase + Ly::kKQ + sm4 * 32768);
            if (lane == 0) mbar_arrive(&bars[kbWReady]);
            if (t == 0) KDA_TRACE1(m, 8);
            return true;
        };
        // Iteration i prepares item i (while there is one) and then converts
        // item i-2: the conversion waits for that item's solve and W product,
        // and lagging it two items keeps the preps (which the next solves
        // wait for) off that path.  The end marker stops the preps; two more
        // passes convert the last items.  One call site each keeps the code
        // small.
        int n_items = 0;
        bool more = true;
#pragma unroll 1
        for (int i = 0;; ++i) {
            if (more) {
                const int s = i % kKqStages, si = i % kKiStages;
                const bool w = t != 0 || wait_or_abort(&bars[kbRawFull + s], (i / kKqStages) & 1,
                                                       abort_flag, p.status);
                if (named_bar_or(1, kPrepThreads, !w)) break;
                const Item it = items[s];
                if (it.m < 0) {   // pass the end on
                    more = false;
                } else {
                    if (t == 0) KDA_TRACE1(i, 1);
                    float *scratch = reinterpret_cast<float *>(sm + Ly::kKI + si * 16384);
                    prep_chunk<true>(t, sbase + Ly::kKQ + s * 32768, sbase + Ly::kKI + si * 16384,
                                     scratch, scratch + 16 * 128, sGL + si * 128, sB + s * 64,
                                     p.beta, it.c0, it.L, p.H, it.h, 1, p.status);
                    if (t == 0) KDA_TRACE1(i, 2);
                    n_items = i + 1;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[kbKqFull + s]);
            }
            if (i >= 2 && i - 2 < n_items && !convert(i - 2)) break;
            if (!more && i - 1 >= n_items) break;
        }
    } else if (warp >= kKsSolve0 && warp < kKsSolve0 + 4) {
        // ---------------------------------------------------------- solve
        const int sw = warp - kKsSolve0;
        const int t = tid - kKsSolve0 * 32;
        // One thread waits on each mbarrier and named_bar_or() shares the
        // outcome, so the four warps leave together on a failed wait and never
        // strand one another at a named barrier.
#pragma unroll 1
        for (int i = 0;; ++i) {
            const int s = i % kKqStages, a = i & 1;
            bool ok = t != 0 || wait_or_abort(&bars[kbApFull + a], (i >> 1) & 1, abort_flag, p.status);
            if (named_bar_or(2, kSolveThreads, !ok)) break;
            if (items[s].m < 0) {   // pass the end on, after the store warp has taken
                                    // TbFull's previous phase (TpFree follows it)
                if (t == 0 && (i < 1 || wait_or_abort(&bars[kbTpFree], (i - 1) & 1, abort_flag,
                                                      p.status)))
                    mbar_arrive(&bars[kbTbFull]);
                break;
            }
            tc_fence_after();
            if (t == 0) KDA_TRACE1(i, 4);
            // D_AP -> L (warps 0, 1: rows 0-63) and -> the bf16 P tile (warps
            // 2, 3: rows 64-127), side by side
            if (sw < 2) build_l(sw, lane, tmem, Ly::kTmAP + a * 64, sL, sB + s * 64);
            else write_p(sw, lane, tmem, Ly::kTmAP + a * 64, sbase + Ly::kP);
            tc_fence_before();
            if (named_bar_or(2, kSolveThreads, !ok)) break;
            if (t == 0) mbar_arrive(&bars[kbApFree + a]);
            invert_unit_lower(sw, lane, sL, sT, 2);
            // the previous chunk's Tb|PT tile must have been read
            if (t == 0 && i >= 1) ok = wait_or_abort(&bars[kbTpFree], (i - 1) & 1, abort_flag, p.status);
            if (named_bar_or(2, kSolveThreads, !ok)) break;
            write_tb(sw, lane, sbase + Ly::kTP, sT, sB + s * 64, 2);
            pt_product(sw, lane, sbase + Ly::kP, sbase + Ly::kTP);
            fence_proxy_async();
            named_bar(2, kSolveThreads);
            if (t == 0) mbar_arrive(&bars[kbTbFull]);
            if (t == 0) KDA_TRACE1(i, 5);
        }
    } else if (warp == kKsMma) {
        // ------------------------------ A/P issuer (lane 0), Ki stores (lanes 1-3)
        // Ki and Gam_L are final once the prep is done.  They leave from here,
        // as soon as they are, rather than from the store warp, which works on
        // the products that follow the solve.
        constexpr uint32_t kIdAP = idesc_bf16(128, 64, 0, 0);
#pragma unroll 1
        for (int i = 0;; ++i) {
            const int s = i % kKqStages, si = i % kKiStages, a = i & 1;
            bool ok = true;
            if (lane == 0)
                ok = wait_or_abort(&bars[kbKqFull + s], (i / kKqStages) & 1, abort_flag, p.status);
            if (!__shfl_sync(0xffffffffu, ok, 0)) break;
            const int m = items[s].m;
            if (m < 0) {   // pass the end on, after the same wait a product takes,
                           // so the solve has consumed ApFull[a]'s previous phase
                if (lane == 0 && (i < 2 || wait_or_abort(&bars[kbApFree + a], ((i - 2) >> 1) & 1,
                                                         abort_flag, p.status)))
                    mbar_arrive(&bars[kbApFull + a]);
                break;
            }
            // the product first: the bulk stores block the warp until their
            // copies have read shared memory
            if (lane == 0) {
                const uint32_t kq = sbase + Ly::kKQ + s * 32768;
                const uint64_t d_kq = smem_desc(kq, 16, 1024, kSw128);
                const uint64_t d_ki = smem_desc(sbase + Ly::kKI + si * 16384, 16, 1024, kSw128);
                if (i >= 2)
                    ok = wait_or_abort(&bars[kbApFree + a], ((i - 2) >> 1) & 1, abort_flag, p.status);
                if (ok) {
                    tc_fence_after();
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks)
                        mma_bf16(tmem + Ly::kTmAP + a * 64, d_kq + kmaj_step(ks, 16384),
                                 d_ki + kmaj_step(ks, 8192), kIdAP, ks > 0);
                    mma_commit(&bars[kbApFull + a]);
                    mma_commit(&bars[kbKiFree + si]);   // the product has read the gate stage
                    KDA_TRACE1(i, 3);
                }
            }
            if (lane >= 1 && lane <= 3) {   // Ki (two 8 KB atoms) and Gam_L, one copy per lane
                if (KDA_IN_RANGE((long long)m < p.slots, p.status)) {
                    unsigned char *dst = p.packets + (size_t)m * kPacketBytes;
                    if (lane < 3)
                        bulk_store(dst + kPkKI + (lane - 1) * 8192,
                                   sm + Ly::kKI + si * 16384 + (lane - 1) * 8192, 8192);
                    else
                        bulk_store(dst + kPkGL, sGL + si * 128, 512);
                    bulk_commit();
                    bulk_wait_read_all();
                }
                mbar_arrive(&bars[kbKiFree + si]);
            }
            if (!__shfl_sync(0xffffffffu, ok, 0)) break;
        }
        if (lane == 0) {
            mma_commit(&bars[kbDrain]);
            mbar_wait(&bars[kbDrain], 0);
        }
        bulk_wait_all();
    }

    KDA_SPAN(g_kda_span1, 1);
    tc_fence_before();
    __syncthreads();
    if (tid == 0) report_abort(abort_flag, p.status);
    if (warp == kKsMma) {
        tc_fence_after();
        tmem_dealloc(tmem, Ly::kTmCols);
    }
}

// ============================================================ pass 2
// Warp roles of the narrow-slice chain pass (32- or 64-column value slices;
// full-width chains take the transposed kernel further down): 4 chain warps
// (warp w keeps rows 32 w .. + 31 of the slice), then the loader and the MMA
// issuer.
template <int VS>
struct ChShape {
    static_assert(VS == 32 || VS == 64, "narrow value slices only");
    static constexpr int kChain = 4;
    static constexpr int kCols = VS;
    static constexpr int kLoad = kChain, kMma = kChain + 1;
    static constexpr int kThreads = (kChain + 2) * 32;
};
enum ChBars {
    cbFull = 0,       // [3] packet + value tile landed (two used when VS = 64)
    cbStageFree = 3,  // [3] every product reading a stage done
    cbSbFull = 6,     // count 4: bf16 S written
    cbUFull = 7,      // D1 = [U; O] complete
    cbUbFull = 8,     // count 2: bf16 U written
    cbDsFull = 9,     // dS = Ki^T U complete
    cbD1Free = 10,    // [2] count 2: O read out of D1[d]
    cbDrain = 12,
    cbNever = 13,     // nothing arrives on it (failure-path check)
    cbNum = 14
};

template <int VS>
struct ChLayout {
    // stage: the packet exactly as stored ([-W; Qe] | Ki | [Tb; PT] | Gam_L),
    // so one bulk copy fills it, then the V slice
    static constexpr uint32_t kKQ = kPkKQ, kKI = kPkKI, kTP = kPkTP, kGL = kPkGL;
    static constexpr uint32_t kV = (kPkGL + 512 + 1023) / 1024 * 1024;
    static constexpr uint32_t kStage = (kV + 64 * VS * 2 + 1023) / 1024 * 1024;
    static_assert(kPkGL + 512 == kPacketBytes, "the packet is one contiguous copy");
    // three stages fit beside the 32-wide operands, two beside the wider ones
    static constexpr int kStages = VS == 32 ? 3 : 2;
    static constexpr uint32_t kSB = kStages * kStage;
    static constexpr uint32_t kUB = kSB + 128 * VS * 2;
    static constexpr uint32_t kBar = kUB + 64 * VS * 2;
    static constexpr uint32_t kMisc = kBar + 16 * 8;
    static constexpr uint32_t kAlloc = kMisc + 16 + 1024;
    static_assert(kAlloc <= 232448, "shared memory budget exceeded");
    static constexpr uint32_t kTmD1 = 0;          // + d * VS, d = chunk & 1
    static constexpr uint32_t kTmD2 = 2 * VS;
    static constexpr uint32_t kTmCols = 4 * VS;   // D1[2], D2, rounded to a power of two
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
    const void *v_base;          // v [T, H, Dv], for the value tile map
    float *snap_pool;            // [snap_slots, H, Dk, Dv] fp32, or null
    const int32_t *snap_base;    // [N] first snapshot slot per sequence, or null
    const int32_t *s0_slot;      // [N] start slot per sequence, or null
    long long snap_slots;
    int snap_every;              // chunks between snapshots; 0: none
    float *ckpt;                 // [packet slots, Dk, Dv] fp32: the state entering every chunk, or null
    int test_stall;              // MMA issuer first waits on cbNever
    int N, T, H;
};

// One CTA per (sequence, head, VS-wide slice of the value dimension) walks
// the sequence's chunks in order.  Per chunk, with S the bf16 copy of the
// fp32 state slice kept in the chain warps' registers:
//   D1  = [Tb; PT] V          (rows 0-63: U0 = Tb V, rows 64-127: P U0)
//   D1 += [-W; Qe] S          (rows 0-63: U,  rows 64-127: O)
//   dS  = Ki^T bf16(U)
//   S   = Diag(Gam_L) (S + dS)
// Only the last two steps and the product of the bf16 S with [-W; Qe] lie on
// the chain from one chunk's state to the next.
template <int VS>
__global__ void __launch_bounds__(ChShape<VS>::kThreads, 1)
chain_kernel(const __grid_constant__ CUtensorMap tm_v, ChParams p) {
    using Ly = ChLayout<VS>;
    using Sh = ChShape<VS>;
    constexpr int kChLoad = Sh::kLoad, kChMma = Sh::kMma, NC = Sh::kCols;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(sm);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + Ly::kBar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + Ly::kMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + Ly::kMisc + 4);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // Launched as a programmatic dependent of the key-side pass: every
    // packet (and the work order) is read only after that pass is done.
    grid_dependency_wait();
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
    const size_t sbase_g = ((size_t)seq * p.H + h) * kDK * kDV + (size_t)vs * VS;

    if (tid == 0) {
        for (int i = 0; i < cbNum; ++i) {
            uint32_t cnt = 1;
            if (i == cbSbFull) cnt = Sh::kChain;
            if (i == cbUbFull || i == cbD1Free || i == cbD1Free + 1) cnt = Sh::kChain / 2;
            mbar_init(&bars[i], cnt);
        }
        abort_flag[0] = 0;
        abort_flag[1] = 0;
        fence_mbar_init();
    }
    if (warp == kChLoad && lane == 0) prefetch_tmap(&tm_v);
    if (warp == kChMma) {
        tmem_alloc(tmem_slot, Ly::kTmCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    KDA_SPAN(g_kda_span2, 0);

    auto packet = [&](int j) {
        return p.packets + ((size_t)(g0 + j) * p.H + h) * kPacketBytes;
    };

    if (warp == kChLoad) {
        // ------------------------------------------------------- loader
        // One copy for the packet (lane 0) and one for the value tile (lane
        // 1): copies from different threads are serviced concurrently.
        int n_issued = 0;
#pragma unroll 1
        for (int j = 0; j < nchunks; ++j) {
            const int s = j % Ly::kStages;
            bool ok = true;
            if (lane == 0 && j >= Ly::kStages)
                ok = wait_or_abort(&bars[cbStageFree + s], (j / Ly::kStages - 1) & 1, abort_flag, p.status);
            if (!__shfl_sync(0xffffffffu, ok, 0)) break;
            unsigned char *st = sm + s * Ly::kStage;
            uint64_t *full = &bars[cbFull + s];
            if (lane == 0) mbar_arrive_expect_tx(full, (uint32_t)kPacketBytes + 64 * VS * 2);
            __syncwarp();
            if (lane < 4) {   // the packet in four pieces, one per lane
                const uint32_t off = lane * 16384u;
                const uint32_t len = lane < 3 ? 16384u : (uint32_t)kPacketBytes - 3 * 16384u;
                bulk_load(st + off, packet(j) + off, len, full);
            }
            if (lane == 4) tma_load_3d(st + Ly::kV, &tm_v, full, vs * VS, h, t0 + j * kChunk);
            if (j + Ly::kStages < nchunks) {   // warm L2 for the copies of chunk j + kStages
                if (lane == 5) bulk_prefetch_l2(packet(j + Ly::kStages), (uint32_t)kPacketBytes);
                if (lane == 8) tma_prefetch_3d(&tm_v, vs * VS, h, t0 + (j + Ly::kStages) * kChunk);
            }
            n_issued = j + 1;
            if (lane == 0) KDA_TRACE2(j, 0);
#ifdef KDA_TRACE
            if (lane == 6) {
                mbar_wait(full, (j / Ly::kStages) & 1);
                KDA_TRACE2(j, 11);
            }
#endif
        }
        // copies in flight must land before the CTA may exit
        if (lane == 0)
            for (int j = max(0, n_issued - Ly::kStages); j < n_issued; ++j)
                mbar_wait(&bars[cbFull + j % Ly::kStages], (j / Ly::kStages) & 1);
    } else if (warp == kChMma) {
        // ------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t kIdV = idesc_bf16(128, VS, 0, 1);
            constexpr uint32_t kIdS = idesc_bf16(128, VS, 1, 1);
            const uint64_t d_sb = vs_desc<VS>(sbase + Ly::kSB, 128);
            const uint64_t d_ub = vs_desc<VS>(sbase + Ly::kUB, 64);
            // D1[d] = [Tb; PT] V for chunk j: issued one chunk ahead, while the
            // chain warps turn the previous chunk's U into bf16, so it never
            // sits between the state and the product that consumes it.
            auto issue_u0 = [&](int j) -> bool {
                const int s = j % Ly::kStages, d = j & 1;
                const uint32_t st = sbase + s * Ly::kStage;
                if (!spin_or_abort(&bars[cbFull + s], (j / Ly::kStages) & 1, abort_flag, p.status))
                    return false;
                KDA_TRACE2(j, 12);
                if (j >= 2 && !spin_or_abort(&bars[cbD1Free + d], ((j - 2) >> 1) & 1, abort_flag,
                                             p.status))
                    return false;
                KDA_TRACE2(j, 1);
                tc_fence_after();
                const uint64_t d_tp = smem_desc(st + Ly::kTP, 16, 1024, kSw128);
                const uint64_t d_v = vs_desc<VS>(st + Ly::kV, 64);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tmem + Ly::kTmD1 + d * VS, d_tp + ((uint64_t)(ks * 32) >> 4),
                             d_v + vs_step<VS>(ks), kIdV, ks > 0);
                return true;
            };
            // failure-path check: a wait that can only run out of time
            bool ok = !p.test_stall || spin_or_abort(&bars[cbNever], 0, abort_flag, p.status);
            ok = ok && nchunks > 0 && issue_u0(0);
#pragma unroll 1
            for (int j = 0; j < nchunks && ok; ++j) {
                const int s = j % Ly::kStages, d = j & 1;
                const uint32_t st = sbase + s * Ly::kStage;
                const uint32_t d1 = tmem + Ly::kTmD1 + d * VS;
                const uint64_t d_kq = smem_desc(st + Ly::kKQ, 16, 1024, kSw128);
                const uint64_t d_kit = smem_desc(st + Ly::kKI, 8192, 1024, kSw128);
                if (!spin_or_abort(&bars[cbSbFull], j & 1, abort_flag, p.status)) break;
                KDA_TRACE2(j, 2);
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)   // D1 += [-W; Qe] S
                    mma_bf16(d1, d_kq + kmaj_step(ks, 16384), d_sb + vs_step<VS>(ks), kIdV, 1);
                mma_commit(&bars[cbUFull]);
                KDA_TRACE2(j, 3);
                // The next chunk's [Tb; PT] V goes in now if its tiles have
                // landed; otherwise after dS, which must not queue behind a
                // copy still in flight.
                bool u0_next = j + 1 >= nchunks;
                if (!u0_next) {
                    const int s1 = (j + 1) % Ly::kStages, d1n = (j + 1) & 1;
                    if (mbar_test_wait(&bars[cbFull + s1], ((j + 1) / Ly::kStages) & 1) &&
                        (j + 1 < 2 || mbar_test_wait(&bars[cbD1Free + d1n], ((j - 1) >> 1) & 1))) {
                        if (!issue_u0(j + 1)) break;
                        u0_next = true;
                    }
                }
                if (!spin_or_abort(&bars[cbUbFull], j & 1, abort_flag, p.status)) break;
                KDA_TRACE2(j, 4);
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)   // dS = Ki^T U
                    mma_bf16(tmem + Ly::kTmD2, d_kit + ((uint64_t)(ks * 2048) >> 4),
                             d_ub + vs_step<VS>(ks), kIdS, ks > 0);
                mma_commit(&bars[cbDsFull]);
                mma_commit(&bars[cbStageFree + s]);
                KDA_TRACE2(j, 5);
                if (!u0_next && !issue_u0(j + 1)) break;
            }
            mma_commit(&bars[cbDrain]);
            mbar_wait(&bars[cbDrain], 0);
        }
    } else {
        // ------------------------------------------------------ chain warps
        const int wq = warp & 3;           // TMEM lane quarter
        const int c = 32 * wq + lane;      // state row (key channel) 0..127
        const int col0 = (warp >> 2) * NC; // this thread's columns of the slice
        float S[NC];
        {
            const float *src = p.S0 ? p.S0 + sbase_g + (size_t)c * kDV + col0 : nullptr;
            if (p.s0_slot) {   // resume from a pool slot (prefix-cache hit)
                const long long slot = p.s0_slot[seq];
                if (slot >= p.snap_slots) {
                    if (c == 0) set_status(p.status, KDA_ERR_SLOT);
                    src = nullptr;
                } else if (slot >= 0) {
                    src = p.snap_pool + ((size_t)slot * p.H + h) * kDK * kDV + (size_t)vs * VS +
                          (size_t)c * kDV + col0;
                }
            }
#pragma unroll
            for (int jj = 0; jj < NC; jj += 4) {
                float4 v = src ? *reinterpret_cast<const float4 *>(src + jj) : make_float4(0, 0, 0, 0);
                S[jj] = v.x; S[jj + 1] = v.y; S[jj + 2] = v.z; S[jj + 3] = v.w;
            }
        }
        float gl_cur = 1.f;
        bool ok = true;
        const long long snap_base = (p.snap_every > 0 && p.snap_base) ? p.snap_base[seq] : -1;
        // snapshot: the state after j >= 1 full chunks, every snap_every chunks
        auto store_snapshot = [&](int j) {
            if (j <= 0 || snap_base < 0 || j % p.snap_every != 0 || j * kChunk > t1 - t0) return;
            const long long slot = snap_base + j / p.snap_every - 1;
            if (slot < p.snap_slots && KDA_IN_RANGE(slot >= 0, p.status)) {
                float *dst = p.snap_pool + ((size_t)slot * p.H + h) * kDK * kDV + (size_t)c * kDV +
                             (size_t)vs * VS + col0;
#pragma unroll
                for (int jj = 0; jj < NC; jj += 4)
                    *reinterpret_cast<float4 *>(dst + jj) =
                        make_float4(S[jj], S[jj + 1], S[jj + 2], S[jj + 3]);
            } else if (c == 0) {
                set_status(p.status, KDA_ERR_SLOT);
            }
        };
#pragma unroll 1
        for (int j = 0; j <= nchunks && ok; ++j) {
            if (j > 0) {
                // S <- Diag(Gam_L) (S + dS) for chunk j-1
                if (!spin_or_abort(&bars[cbDsFull], (j - 1) & 1, abort_flag, p.status)) { ok = false; break; }
                tc_fence_after();
                if (c == 0) KDA_TRACE2(j - 1, 6);
#pragma unroll
                for (int jj = 0; jj < NC; jj += 32) {
                    uint32_t v[32];
                    tmem_ld32(tmem_addr(tmem, 32 * wq, Ly::kTmD2 + col0 + jj), v);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) S[jj + e] = gl_cur * (S[jj + e] + __uint_as_float(v[e]));
                }
            }
            if (j == nchunks) {
                store_snapshot(j);
                break;
            }
            const int s = j % Ly::kStages, d = j & 1;
            if (!spin_or_abort(&bars[cbFull + s], (j / Ly::kStages) & 1, abort_flag, p.status)) { ok = false; break; }
            gl_cur = reinterpret_cast<const float *>(sm + s * Ly::kStage + Ly::kGL)[c];
            if (c == 0) KDA_TRACE2(j, 7);
            {
                const uint32_t sb = sbase + Ly::kSB;
#pragma unroll
                for (int q8 = 0; q8 < NC / 8; ++q8) {
                    sts128(sb + vs_off<VS>(c, col0 / 8 + q8, 128), pack2(S[8 * q8], S[8 * q8 + 1]),
                           pack2(S[8 * q8 + 2], S[8 * q8 + 3]), pack2(S[8 * q8 + 4], S[8 * q8 + 5]),
                           pack2(S[8 * q8 + 6], S[8 * q8 + 7]));
                }
            }
            fence_proxy_async();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[cbSbFull]);
            if (c == 0) KDA_TRACE2(j, 8);
            // the state entering chunk j, for the chunked backward: stored after
            // the proxy fence above so that fence never waits for it
            if (p.ckpt && KDA_IN_RANGE(((long long)g0 + j) * p.H + h < p.slots, p.status)) {
                float *dst = p.ckpt + ((size_t)(g0 + j) * p.H + h) * kDK * kDV + (size_t)c * kDV +
                             (size_t)vs * VS + col0;
#pragma unroll
                for (int jj = 0; jj < NC; jj += 4)
                    *reinterpret_cast<float4 *>(dst + jj) =
                        make_float4(S[jj], S[jj + 1], S[jj + 2], S[jj + 3]);
            }
            // Snapshot stores go after a proxy fence, never just before one: the
            // fence would wait for them to complete.  Rows 64-127 next fence a
            // chunk later; rows 0-63 fence the U operand below, so they store
            // after that.
            if (j > 0 && wq >= 2) store_snapshot(j);

            if (!spin_or_abort(&bars[cbUFull], j & 1, abort_flag, p.status)) { ok = false; break; }
            tc_fence_after();
            if (wq < 2) {
                // U rows: D1 lanes 0..63 -> bf16 operand of dS
                if (c == 0) KDA_TRACE2(j, 9);
                const uint32_t ub = sbase + Ly::kUB;
#pragma unroll
                for (int jj = 0; jj < NC; jj += 32) {
                    uint32_t v[32];
                    tmem_ld32(tmem_addr(tmem, 32 * wq, Ly::kTmD1 + d * VS + col0 + jj), v);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; e += 8) {
                        sts128(ub + vs_off<VS>(c, (col0 + jj + e) / 8, 64),
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
                if (j > 0) store_snapshot(j);
            } else {
                // O rows: D1 lanes 64..127 -> bf16 output, once U is converted:
                // these global stores share the load/store pipe with the U rows'
                // shared-memory stores on the chain's critical path
                if (!wait_or_abort(&bars[cbUbFull], j & 1, abort_flag, p.status)) { ok = false; break; }
                const int c0 = t0 + j * kChunk, L = min(kChunk, t1 - c0);
                const int r = c - 64;
#pragma unroll
                for (int jj = 0; jj < NC; jj += 32) {
                    uint32_t v[32];
                    tmem_ld32(tmem_addr(tmem, 32 * wq, Ly::kTmD1 + d * VS + col0 + jj), v);
                    tmem_wait_ld();
                    if (r < L && p.out && KDA_IN_RANGE(c0 + r < p.T, p.status)) {
                        __nv_bfloat16 *dst =
                            p.out + ((size_t)(c0 + r) * p.H + h) * kDV + vs * VS + col0 + jj;
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
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[cbD1Free + d]);
            }
        }
        if (ok && p.Sf && KDA_IN_RANGE(seq < p.N, p.status)) {
            float *dst = p.Sf + sbase_g + (size_t)c * kDV + col0;
#pragma unroll
            for (int jj = 0; jj < NC; jj += 4)
                *reinterpret_cast<float4 *>(dst + jj) = make_float4(S[jj], S[jj + 1], S[jj + 2], S[jj + 3]);
        }
    }

    KDA_SPAN(g_kda_span2, 1);
    tc_fence_before();
    __syncthreads();
    if (tid == 0) report_abort(abort_flag, p.status);
    if (warp == kChMma) {
        tc_fence_after();
        tmem_dealloc(tmem, Ly::kTmCols);
    }
}

// ------------------------------------------------ pass 2, transposed chain
// For full-width (128-column) value slices the chain runs transposed, with
// TMEM lane = value column v:
//   D1^T  = V^T [Tb; PT]^T        (columns 0-63: U^T, 64-127: P U0 parts)
//   D1^T += S^T [-W; Qe]^T        (columns 0-63: U^T, 64-127: O^T)
//   dS^T  = U^T Ki ;  S^T <- (S^T + dS^T) Diag(Gam_L)
// S^T (bf16) and U^T (bf16) are the A operands of the two products on the
// chain and go to tensor memory with tcgen05.st, so nothing on the chain
// passes through shared memory except the packet and V tiles, which every
// product reads as its B operand (or A, for V^T) exactly as they landed.
// Warp w (of 8) keeps lane quarter w % 4 (v = 32 (w % 4) + lane) and half
// w / 4: key channels 64 (w / 4) .. + 63 of the state, positions
// 32 (w / 4) .. + 31 of U and O.
constexpr int kCtChain = 8, kCtLoad = 8, kCtMma = 9, kCtThreads = 10 * 32;
struct ChTLayout {
    static constexpr uint32_t kKQ = kPkKQ, kKI = kPkKI, kTP = kPkTP, kGL = kPkGL;
    static constexpr uint32_t kV = (kPkGL + 512 + 1023) / 1024 * 1024;   // two 64-column atoms
    static constexpr uint32_t kStage = (kV + 64 * 128 * 2 + 1023) / 1024 * 1024;
    static constexpr int kStages = 2;
    static constexpr uint32_t kOS = kStages * kStage;   // 8 x [32 positions][32 columns] bf16
    static constexpr uint32_t kBar = kOS + kCtChain * 2048;
    static constexpr uint32_t kMisc = kBar + 16 * 8;
    static constexpr uint32_t kAlloc = kMisc + 16 + 1024;
    static_assert(kAlloc <= 232448, "shared memory budget exceeded");
    static constexpr uint32_t kTmD1 = 0;     // + 128 d, d = chunk & 1
    static constexpr uint32_t kTmD2 = 256;   // dS^T, 128 columns
    static constexpr uint32_t kTmAS = 384;   // S^T as bf16 pairs, 64 columns
    static constexpr uint32_t kTmAU = 448;   // U^T as bf16 pairs, 32 columns
    static constexpr uint32_t kTmCols = 512;
};

__global__ void __launch_bounds__(kCtThreads, 1)
chain_t_kernel(const __grid_constant__ CUtensorMap tm_v, ChParams p) {
    using Ly = ChTLayout;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(sm);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + Ly::kBar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + Ly::kMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + Ly::kMisc + 4);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // a programmatic dependent of the key-side pass: packets and the work
    // order are read only after that pass is done
    grid_dependency_wait();
    const int seq = p.order[blockIdx.x / p.H];
    const int h = blockIdx.x % p.H;
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
    const size_t sbase_g = ((size_t)seq * p.H + h) * kDK * kDV;

    if (tid == 0) {
        for (int i = 0; i < cbNum; ++i) {
            uint32_t cnt = 1;
            if (i == cbSbFull || i == cbUbFull || i == cbD1Free || i == cbD1Free + 1) cnt = kCtChain;
            if (i >= cbStageFree && i < cbStageFree + Ly::kStages) cnt = 1 + kCtChain;
            mbar_init(&bars[i], cnt);
        }
        abort_flag[0] = 0;
        abort_flag[1] = 0;
        fence_mbar_init();
    }
    if (warp == kCtLoad && lane == 0) prefetch_tmap(&tm_v);
    if (warp == kCtMma) {
        tmem_alloc(tmem_slot, Ly::kTmCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    KDA_SPAN(g_kda_span2, 0);

    auto packet = [&](int j) {
        return p.packets + ((size_t)(g0 + j) * p.H + h) * kPacketBytes;
    };

    if (warp == kCtLoad) {
        // ------------------------------------------------------- loader
        int n_issued = 0;
#pragma unroll 1
        for (int j = 0; j < nchunks; ++j) {
            const int s = j % Ly::kStages;
            bool ok = true;
            if (lane == 0 && j >= Ly::kStages)
                ok = wait_or_abort(&bars[cbStageFree + s], (j / Ly::kStages - 1) & 1, abort_flag, p.status);
            if (!__shfl_sync(0xffffffffu, ok, 0)) break;
            unsigned char *st = sm + s * Ly::kStage;
            uint64_t *full = &bars[cbFull + s];
            if (lane == 0) mbar_arrive_expect_tx(full, (uint32_t)kPacketBytes + 64 * 128 * 2);
            __syncwarp();
            if (lane < 4) {   // the packet in four pieces, one per lane
                const uint32_t off = lane * 16384u;
                const uint32_t len = lane < 3 ? 16384u : (uint32_t)kPacketBytes - 3 * 16384u;
                bulk_load(st + off, packet(j) + off, len, full);
            }
            if (lane == 4) tma_load_3d(st + Ly::kV, &tm_v, full, 0, h, t0 + j * kChunk);
            if (lane == 7) tma_load_3d(st + Ly::kV + 64 * 128, &tm_v, full, 64, h, t0 + j * kChunk);
            if (j + Ly::kStages < nchunks) {   // warm L2 for the copies of chunk j + 2
                if (lane == 5) bulk_prefetch_l2(packet(j + Ly::kStages), (uint32_t)kPacketBytes);
                if (lane == 8) tma_prefetch_3d(&tm_v, 0, h, t0 + (j + Ly::kStages) * kChunk);
                if (lane == 9) tma_prefetch_3d(&tm_v, 64, h, t0 + (j + Ly::kStages) * kChunk);
            }
            n_issued = j + 1;
            if (lane == 0) KDA_TRACE2(j, 0);
#ifdef KDA_TRACE
            if (lane == 6) {
                mbar_wait(full, (j / Ly::kStages) & 1);
                KDA_TRACE2(j, 11);
            }
#endif
        }
        if (lane == 0)
            for (int j = max(0, n_issued - Ly::kStages); j < n_issued; ++j)
                mbar_wait(&bars[cbFull + j % Ly::kStages], (j / Ly::kStages) & 1);
    } else if (warp == kCtMma) {
        // ------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t kIdU0 = idesc_bf16(128, 128, 1, 0);   // V^T (MN-major) x [Tb;PT]^T
            constexpr uint32_t kIdS = idesc_bf16(128, 128, 0, 0);    // S^T (TMEM) x [-W;Qe]^T
            constexpr uint32_t kIdDs = idesc_bf16(128, 128, 0, 1);   // U^T (TMEM) x Ki (MN-major)
            auto issue_u0 = [&](int j) -> bool {
                const int s = j % Ly::kStages, d = j & 1;
                const uint32_t st = sbase + s * Ly::kStage;
                if (!spin_or_abort(&bars[cbFull + s], (j / Ly::kStages) & 1, abort_flag, p.status))
                    return false;
                KDA_TRACE2(j, 12);
                if (j >= 2 && !spin_or_abort(&bars[cbD1Free + d], ((j - 2) >> 1) & 1, abort_flag,
                                             p.status))
                    return false;
                KDA_TRACE2(j, 1);
                tc_fence_after();
                const uint64_t d_v = smem_desc(st + Ly::kV, 64 * 128, 1024, kSw128);
                const uint64_t d_tp = smem_desc(st + Ly::kTP, 16, 1024, kSw128);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tmem + Ly::kTmD1 + d * 128, d_v + ((uint64_t)(ks * 2048) >> 4),
                             d_tp + ((uint64_t)(ks * 32) >> 4), kIdU0, ks > 0);
                return true;
            };
            bool ok = !p.test_stall || spin_or_abort(&bars[cbNever], 0, abort_flag, p.status);
            ok = ok && nchunks > 0 && issue_u0(0);
#pragma unroll 1
            for (int j = 0; j < nchunks && ok; ++j) {
                const int s = j % Ly::kStages, d = j & 1;
                const uint32_t st = sbase + s * Ly::kStage;
                const uint32_t d1 = tmem + Ly::kTmD1 + d * 128;
                if (!spin_or_abort(&bars[cbSbFull], j & 1, abort_flag, p.status)) break;
                KDA_TRACE2(j, 2);
                tc_fence_after();
                const uint64_t d_kq = smem_desc(st + Ly::kKQ, 16, 1024, kSw128);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)   // D1^T += S^T [-W; Qe]^T
                    mma_bf16_ta(d1, tmem + Ly::kTmAS + 8 * ks, d_kq + kmaj_step(ks, 16384), kIdS, 1);
                mma_commit(&bars[cbUFull]);
                KDA_TRACE2(j, 3);
                // the next chunk's V^T [Tb; PT]^T now if its tiles have landed,
                // otherwise after dS
                bool u0_next = j + 1 >= nchunks;
                if (!u0_next) {
                    const int s1 = (j + 1) % Ly::kStages, d1n = (j + 1) & 1;
                    if (mbar_test_wait(&bars[cbFull + s1], ((j + 1) / Ly::kStages) & 1) &&
                        (j + 1 < 2 || mbar_test_wait(&bars[cbD1Free + d1n], ((j - 1) >> 1) & 1))) {
                        if (!issue_u0(j + 1)) break;
                        u0_next = true;
                    }
                }
                if (!spin_or_abort(&bars[cbUbFull], j & 1, abort_flag, p.status)) break;
                KDA_TRACE2(j, 4);
                tc_fence_after();
                const uint64_t d_ki = smem_desc(st + Ly::kKI, 64 * 128, 1024, kSw128);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)   // dS^T = U^T Ki
                    mma_bf16_ta(tmem + Ly::kTmD2, tmem + Ly::kTmAU + 8 * ks,
                                d_ki + ((uint64_t)(ks * 2048) >> 4), kIdDs, ks > 0);
                mma_commit(&bars[cbDsFull]);
                mma_commit(&bars[cbStageFree + s]);
                KDA_TRACE2(j, 5);
                if (!u0_next && !issue_u0(j + 1)) break;
            }
            mma_commit(&bars[cbDrain]);
            mbar_wait(&bars[cbDrain], 0);
        }
    } else {
        // ------------------------------------------------------ chain warps
        const int wq = warp & 3, hf = warp >> 2;
        const int v = 32 * wq + lane;           // value column (TMEM lane)
        const int cb = 64 * hf;                 // first key channel of this thread's state
        float S[64];                            // S[c] = state[cb + c][v]
        {
            const float *src = p.S0 ? p.S0 + sbase_g : nullptr;
            if (p.s0_slot) {   // resume from a pool slot (prefix-cache hit)
                const long long slot = p.s0_slot[seq];
                if (slot >= p.snap_slots) {
                    if (tid == 0) set_status(p.status, KDA_ERR_SLOT);
                    src = nullptr;
                } else if (slot >= 0) {
                    src = p.snap_pool + ((size_t)slot * p.H + h) * kDK * kDV;
                }
            }
#pragma unroll
            for (int c = 0; c < 64; ++c) S[c] = src ? src[(size_t)(cb + c) * kDV + v] : 0.f;
        }
        auto store_state = [&](float *dst) {   // dst: a [Dk][Dv] state
#pragma unroll
            for (int c = 0; c < 64; ++c) dst[(size_t)(cb + c) * kDV + v] = S[c];
        };
        bool ok = true;
        const long long snap_base = (p.snap_every > 0 && p.snap_base) ? p.snap_base[seq] : -1;
        auto store_snapshot = [&](int j) {
            if (j <= 0 || snap_base < 0 || j % p.snap_every != 0 || j * kChunk > t1 - t0) return;
            const long long slot = snap_base + j / p.snap_every - 1;
            if (slot < p.snap_slots && KDA_IN_RANGE(slot >= 0, p.status))
                store_state(p.snap_pool + ((size_t)slot * p.H + h) * kDK * kDV);
            else if (tid == 0)
                set_status(p.status, KDA_ERR_SLOT);
        };
#pragma unroll 1
        for (int j = 0; j <= nchunks && ok; ++j) {
            if (j > 0) {
                // S^T <- (S^T + dS^T) Diag(Gam_L) for chunk j-1; then its stage
                // may be refilled
                const int sp = (j - 1) % Ly::kStages;
                if (!spin_or_abort(&bars[cbDsFull], (j - 1) & 1, abort_flag, p.status)) { ok = false; break; }
                if (tid == 0) KDA_TRACE2(j - 1, 6);
                tc_fence_after();
                const float4 *gl = reinterpret_cast<const float4 *>(sm + sp * Ly::kStage + Ly::kGL) + cb / 4;
#pragma unroll
                for (int jj = 0; jj < 64; jj += 32) {
                    uint32_t dv[32];
                    tmem_ld32(tmem_addr(tmem, 32 * wq, Ly::kTmD2 + cb + jj), dv);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; e += 4) {
                        const float4 g = gl[(jj + e) / 4];
                        S[jj + e] = g.x * (S[jj + e] + __uint_as_float(dv[e]));
                        S[jj + e + 1] = g.y * (S[jj + e + 1] + __uint_as_float(dv[e + 1]));
                        S[jj + e + 2] = g.z * (S[jj + e + 2] + __uint_as_float(dv[e + 2]));
                        S[jj + e + 3] = g.w * (S[jj + e + 3] + __uint_as_float(dv[e + 3]));
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[cbStageFree + sp]);
                if (tid == 0) KDA_TRACE2(j - 1, 14);
            }
            if (j == nchunks) {
                store_snapshot(j);
                break;
            }
            const int s = j % Ly::kStages, d = j & 1;
            if (!spin_or_abort(&bars[cbFull + s], (j / Ly::kStages) & 1, abort_flag, p.status)) { ok = false; break; }
            if (tid == 0) KDA_TRACE2(j, 7);
            {   // S^T as bf16 pairs -> the A operand of D1^T += S^T [-W; Qe]^T
#pragma unroll
                for (int jj = 0; jj < 64; jj += 32) {
                    uint32_t w[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) w[e] = pack2(S[jj + 2 * e], S[jj + 2 * e + 1]);
                    tmem_st16(tmem_addr(tmem, 32 * wq, Ly::kTmAS + cb / 2 + jj / 2), w);
                }
                tmem_wait_st();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[cbSbFull]);
            if (tid == 0) KDA_TRACE2(j, 8);
            // the state entering chunk j, for the chunked backward
            if (p.ckpt && KDA_IN_RANGE(((long long)g0 + j) * p.H + h < p.slots, p.status))
                store_state(p.ckpt + ((size_t)(g0 + j) * p.H + h) * kDK * kDV);
            if (j > 0) store_snapshot(j);

            if (!spin_or_abort(&bars[cbUFull], j & 1, abort_flag, p.status)) { ok = false; break; }
            if (tid == 0) KDA_TRACE2(j, 9);
            tc_fence_after();
            {   // U^T positions 32 hf .. + 31 -> bf16 pairs, the A operand of dS^T
                uint32_t u[32];
                tmem_ld32(tmem_addr(tmem, 32 * wq, Ly::kTmD1 + d * 128 + 32 * hf), u);
                tmem_wait_ld();
                uint32_t w[16];
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    w[e] = pack2(__uint_as_float(u[2 * e]), __uint_as_float(u[2 * e + 1]));
                tmem_st16(tmem_addr(tmem, 32 * wq, Ly::kTmAU + 16 * hf), w);
                tmem_wait_st();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[cbUbFull]);
            if (tid == 0) KDA_TRACE2(j, 10);
            {   // O^T positions 32 hf .. + 31, columns 32 wq .. + 31 -> bf16 output
                // rows, through a per-warp transpose in shared memory so that the
                // global stores are 16-byte
                const int c0 = t0 + j * kChunk, L = min(kChunk, t1 - c0);
                uint32_t o[32];
                tmem_ld32(tmem_addr(tmem, 32 * wq, Ly::kTmD1 + d * 128 + 64 + 32 * hf), o);
                tmem_wait_ld();
                const uint32_t ob = sbase + Ly::kOS + warp * 2048;
#pragma unroll
                for (int e = 0; e < 32; ++e) sts16(ob + e * 64 + lane * 2, bf16_bits(__uint_as_float(o[e])));
                __syncwarp();
                if (p.out) {
#pragma unroll
                    for (int r4 = 0; r4 < 4; ++r4) {
                        const int e = (lane >> 2) + 8 * r4, vg = lane & 3, r = 32 * hf + e;
                        const uint4 val = lds128(ob + e * 64 + vg * 16);
                        if (r < L && KDA_IN_RANGE(c0 + r < p.T, p.status))
                            *reinterpret_cast<uint4 *>(p.out + ((size_t)(c0 + r) * p.H + h) * kDV +
                                                       32 * wq + 8 * vg) = val;
                    }
                }
                __syncwarp();   // read out before the next chunk's rows land
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[cbD1Free + d]);
            if (tid == 0) KDA_TRACE2(j, 13);
        }
        if (ok && p.Sf && KDA_IN_RANGE(seq < p.N, p.status)) store_state(p.Sf + sbase_g);
    }

    KDA_SPAN(g_kda_span2, 1);
    tc_fence_before();
    __syncthreads();
    if (tid == 0) report_abort(abort_flag, p.status);
    if (warp == kCtMma) {
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

namespace {

// Launch with programmatic stream serialisation: the kernel may start while
// the previous kernel in the stream finishes (it waits for that kernel's
// results itself, see grid_dependency_wait).
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kern)(KArgs...), unsigned grid, unsigned block, size_t smem,
                             cudaStream_t s, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

template <int VS>
cudaError_t launch_chain(const ChParams &cp, int T, cudaStream_t s) {
    CUtensorMap mv;
    if (!make_tmap_bf16_3d(&mv, cp.v_base, T, cp.H, kDV, VS, VS * 2)) return cudaErrorInvalidValue;
    auto kern = chain_kernel<VS>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)ChLayout<VS>::kAlloc);
    if (e != cudaSuccess) return e;
    const unsigned grid2 = (unsigned)cp.N * cp.H * (kDV / VS);
    return launch_dependent(kern, grid2, ChShape<VS>::kThreads, ChLayout<VS>::kAlloc, s, mv, cp);
}

cudaError_t launch_chain_t(const ChParams &cp, int T, cudaStream_t s) {
    CUtensorMap mv;   // the V tile as two 64-column boxes
    if (!make_tmap_bf16_3d(&mv, cp.v_base, T, cp.H, kDV, 64, 128)) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(chain_t_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)ChTLayout::kAlloc);
    if (e != cudaSuccess) return e;
    const unsigned grid2 = (unsigned)cp.N * cp.H;
    return launch_dependent(chain_t_kernel, grid2, kCtThreads, ChTLayout::kAlloc, s, mv, cp);
}

}  // namespace

cudaError_t launch_prefill_two_pass(const ForwardArgs &a, cudaStream_t s) {
    const int T = a.T > 0 ? a.T : 1;
    CUtensorMap mq, mk, mla;
    if (!make_tmap_bf16_3d(&mq, a.q, T, a.H, kDK, 64, 128) ||
        !make_tmap_bf16_3d(&mk, a.k, T, a.H, kDK, 64, 128) ||
        !make_tmap_bf16_3d(&mla, a.log_alpha, T, a.H, kDK, 64, 128))
        return cudaErrorInvalidValue;
    // pass 1: persistent, at most one CTA per SM, items claimed from a counter
    KsParams kp;
    kp.beta = static_cast<const __nv_bfloat16 *>(a.beta);
    kp.cu = a.cu_seqlens;
    kp.chunk_off = a.chunk_off;
    kp.packets = a.packets;
    kp.slots = (long long)a.packet_slots;
    kp.status = a.status;
    kp.work_ctr = a.work_ctr;
    kp.N = a.N;
    kp.H = a.H;
    cudaError_t e = cudaFuncSetAttribute(kside_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)KsLayout::kAlloc);
    if (e != cudaSuccess) return e;
    const size_t items = a.packet_slots;
    const unsigned grid1 = (unsigned)(items < (size_t)sm_count() ? items : (size_t)sm_count());
    if ((e = launch_dependent(kside_kernel, grid1, kKsThreads, KsLayout::kAlloc, s, mq, mk, mla,
                              kp)) != cudaSuccess)
        return e;
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
    cp.snap_pool = a.snap_pool;
    cp.snap_base = a.snap_base;
    cp.s0_slot = a.s0_slot;
    cp.snap_slots = a.snap_slots;
    cp.snap_every = a.snap_every_chunks;
    cp.ckpt = a.ckpt;
    cp.test_stall = a.test_stall ? 1 : 0;
    cp.N = a.N;
    cp.T = a.T;
    cp.H = a.H;
    cp.v_base = a.v;
    // pass 2: one CTA per (sequence, head, value slice), longest sequences
    // first.  32-wide slices give the most parallel chains (the chain is then
    // bound by its per-chunk latency); once they would not fit on the GPU in
    // one wave the pass is bound by shared-memory traffic, which wider slices
    // cut per chunk and head: the packet lands once instead of two or four
    // times, and a wider MMA reads its A operand once for more columns.
    const long long chains = (long long)a.N * a.H;
    if (chains * (kDV / 32) <= sm_count()) return launch_chain<32>(cp, T, s);
    if (chains * (kDV / 64) <= sm_count()) return launch_chain<64>(cp, T, s);
    return launch_chain_t(cp, T, s);
}

}  // namespace kda

#ifdef KDA_TRACE
extern "C" int kda_trace1_read(unsigned long long *host) {
    return (int)cudaMemcpyFromSymbol(host, kda::g_kda_trace1, sizeof(kda::g_kda_trace1));
}
extern "C" int kda_span_read(int which, unsigned long long *host) {
    return (int)(which == 1 ? cudaMemcpyFromSymbol(host, kda::g_kda_span1, sizeof(kda::g_kda_span1))
                            : cudaMemcpyFromSymbol(host, kda::g_kda_span2, sizeof(kda::g_kda_span2)));
}
extern "C" int kda_trace2_read(unsigned long long *host) {
    return (int)cudaMemcpyFromSymbol(host, kda::g_kda_trace2, sizeof(kda::g_kda_trace2));
}
#endif
