// kda_backward.cu -- gradients of the KDA recurrence on CUDA cores, fp32.
//
// The page "Kimi K3: Open Frontier Intelligence and Implementation
// Framework" (section "Hybrid Attention Mechanism", KDA bullet) defines the
// recurrence, per (sequence, head) chain, one token at a time:
//     1. P = Diag(alpha_t) S_{t-1},   alpha_t = exp(log_alpha_t)
//     2. u = v_t - P^T k_t
//     3. S_t = P + beta_t k_t u^T
//     4. o_t = S_t^T q_t
// and the same page trains the model built on it.  Given dL/do_t (d_out) and
// optionally dL/dS_final, this file computes the gradients of L with respect
// to q, k, v, log_alpha, beta and S0 by the chain rule through those steps in
// reverse order.  With G = dL/dS_t on entry to token t:
//     4'. dq_t = S_t do_t;                      G += q_t do_t^T
//     3'. du = beta G^T k;  dk_t = beta G u;    dbeta_t = k^T G u;   dP = G
//     2'. dv_t = du;        dP -= k du^T;       dk_t -= P du
//     1'. dlog_alpha_t = alpha_t * rowsum(dP * S_{t-1});  G = Diag(alpha_t) dP
// and dS0 = G after the chain's first token.
//
// Work decomposition.  Steps 1-3 act on the columns of S independently, and
// so do 1'-3' on the columns of G, so one CTA takes one (sequence, head,
// 32-wide value slice); thread c holds row c of the slice of S and of G (32
// fp32 registers each).  The per-column sums over the rows (P^T k and G^T k)
// are one butterfly reduce-scatter per warp plus a sum over the warps in
// shared memory.  The per-row sums over the columns (dq, dk, dlog_alpha) and
// dbeta get one partial sum per slice: each slice stores its own in the
// workspace and a second kernel adds the slices in slice order, so every
// gradient is the same fixed sequence of fp32 operations on every call
// (bitwise reproducible; no atomics).
//
// States: pass A runs the chain forward and stores the state every kBwStep =
// 32 tokens (a "step").  Pass B walks the steps backward; for each it
// recomputes the step's 32 states from its checkpoint into a per-CTA scratch
// (with u of every token), then runs the reverse steps over them.  The
// forward is thus evaluated twice and every state is exact fp32 recomputation,
// not an inverse of the recurrence.  32 tokens keep the scratch of all CTAs
// (512 KB each at d = 128) inside L2.
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kBwVs = 32;   // value columns per CTA

struct BwParams {
    const void *q, *k, *v, *la, *beta, *d_out;
    const float *S0, *dSf;
    const int32_t *cu, *order, *chunk_off;
    float *dq, *dk, *dv, *dla, *dbeta, *dS0;
    float *ckpt;             // [ckpt_steps, H, n_slices, DK, 32]
    float *scratch;          // per CTA: [kBwStep, DK, 32] states, then [kBwStep, 32] u
    float *part;             // per slice: dq, dk, dlog_alpha [T, H, DK], dbeta [T, H]
    size_t part_stride;      // floats per slice of `part`
    long long ckpt_steps;    // checkpoints the workspace holds (per head and slice)
    int32_t *status;
    int N, T, H, Dv;
};

// 32 consecutive elements -> fp32 registers (16-byte vector loads).
__device__ __forceinline__ void load32(const float *src, float (&x)[32]) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float4 w = reinterpret_cast<const float4 *>(src)[i];
        x[4 * i] = w.x; x[4 * i + 1] = w.y; x[4 * i + 2] = w.z; x[4 * i + 3] = w.w;
    }
}
__device__ __forceinline__ void load32(const __nv_bfloat16 *src, float (&x)[32]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint4 w = reinterpret_cast<const uint4 *>(src)[i];
        const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            x[8 * i + 2 * e] = __uint_as_float(wv[e] << 16);
            x[8 * i + 2 * e + 1] = __uint_as_float(wv[e] & 0xFFFF0000u);
        }
    }
}
__device__ __forceinline__ void store32(float *dst, const float (&x)[32]) {
#pragma unroll
    for (int i = 0; i < 8; ++i)
        reinterpret_cast<float4 *>(dst)[i] =
            make_float4(x[4 * i], x[4 * i + 1], x[4 * i + 2], x[4 * i + 3]);
}

// Butterfly reduce-scatter: returns, in lane l, the sum over the warp's lanes
// of x[l].  Stage s halves the values a lane keeps (x is consumed).
__device__ __forceinline__ float lane_column_sum(float (&x)[32], int lane) {
#pragma unroll
    for (int s = 16; s >= 1; s >>= 1) {
        const bool up = (lane & s) != 0;
#pragma unroll
        for (int i = 0; i < s; ++i) {
            const float send = up ? x[i] : x[i + s];
            const float keep = up ? x[i + s] : x[i];
            x[i] = keep + __shfl_xor_sync(0xffffffffu, send, s);
        }
    }
    return x[0];
}

// Pull the 128-byte line holding `p` into L1 (and L2) ahead of its load.
__device__ __forceinline__ void prefetch_l1(const void *p) {
    asm volatile("prefetch.global.L1 [%0];" ::"l"(p));
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int s = 16; s >= 1; s >>= 1) x += __shfl_xor_sync(0xffffffffu, x, s);
    return x;
}

template <typename TIO, typename TG, int DK>
__global__ void __launch_bounds__(DK)
backward_kernel(BwParams p) {
    constexpr int NW = DK / 32;
    __shared__ __align__(16) float red[2][NW][32];   // per-warp column sums, by round parity
    __shared__ float redb[2][NW];                    // per-warp dbeta partial sums

    const TIO *q = static_cast<const TIO *>(p.q), *k = static_cast<const TIO *>(p.k);
    const TIO *v = static_cast<const TIO *>(p.v), *dout = static_cast<const TIO *>(p.d_out);
    const TG *la = static_cast<const TG *>(p.la), *beta = static_cast<const TG *>(p.beta);

    const int c = threadIdx.x, warp = c >> 5, lane = c & 31;
    const int n_slices = p.Dv / kBwVs;
    const int per_seq = p.H * n_slices;
    const int n = p.order[blockIdx.x / per_seq];
    const int h = (blockIdx.x % per_seq) / n_slices;
    const int vs = blockIdx.x % n_slices;
    int t0, t1;
    if (!seq_range(p.cu, n, p.T, t0, t1)) {
        if (c == 0) set_status(p.status, KDA_ERR_SEQLENS);
        return;
    }
    // sequence n's steps take checkpoint slots 2 chunk_off[n] .. + ceil(len / 32)
    // (at most two per 64-token chunk)
    const int nc = (t1 - t0 + kBwStep - 1) / kBwStep;
    const long long g0 = 2LL * p.chunk_off[n];
    if (g0 + nc > p.ckpt_steps) {   // overlapping (malformed) sequences
        if (c == 0) set_status(p.status, KDA_ERR_SEQLENS);
        return;
    }
    const size_t col0 = (size_t)vs * kBwVs;
    auto ckpt_row = [&](int j) {
        return p.ckpt + ((((size_t)g0 + j) * p.H + h) * n_slices + vs) * DK * kBwVs +
               (size_t)c * kBwVs;
    };
    float *scr = p.scratch + (size_t)blockIdx.x * (kBwStep * DK * kBwVs + kBwStep * kBwVs);
    // this slice's partial row sums
    const size_t thd = (size_t)p.T * p.H * DK;
    float *part_dq = p.part + (size_t)vs * p.part_stride;
    float *part_dk = part_dq + thd, *part_dla = part_dq + 2 * thd, *part_db = part_dq + 3 * thd;
    float *scr_u = scr + kBwStep * DK * kBwVs;
    int round = 0;

    // u = v_t - (Diag(alpha) S)^T k_t for this slice, S <- Diag(alpha) S + beta k u^T.
    // Column j of u, from the round's shared sums, is the same expression
    // (the warps' sums added in warp order) wherever it is formed.
    auto col_sum = [&](int par, int j) {
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) s += red[par][w][j];
        return s;
    };
    // all 32 column sums: lane l forms column l's, then the warp shares them
    auto col_sums = [&](int par, float (&cs)[32]) {
        const float mine = col_sum(par, lane);
#pragma unroll
        for (int j = 0; j < 32; ++j) cs[j] = __shfl_sync(0xffffffffu, mine, j);
    };
    // the inputs of token t: this thread's key row elements and the slice's v / d_out
    auto prefetch_token = [&](int t, bool with_q) {
        const size_t rk = ((size_t)t * p.H + h) * DK + c;
        prefetch_l1(k + rk);
        prefetch_l1(la + rk);
        if (with_q) prefetch_l1(q + rk);
        if (c == 0) {
            prefetch_l1(beta + (size_t)t * p.H + h);
            prefetch_l1(v + ((size_t)t * p.H + h) * p.Dv + col0);
            if (with_q) prefetch_l1(dout + ((size_t)t * p.H + h) * p.Dv + col0);
        }
    };
    auto forward_token = [&](int t, float (&S)[32], float *u_out) {
        const size_t rk = ((size_t)t * p.H + h) * DK + c;
        if (t + 1 < t1) prefetch_token(t + 1, false);
        const float kc = to_f32(k[rk]), ac = expf(to_f32(la[rk]));
        const float bt = to_f32(beta[(size_t)t * p.H + h]);
        float vv[32], x[32];
        load32(v + ((size_t)t * p.H + h) * p.Dv + col0, vv);
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            S[j] *= ac;
            x[j] = S[j] * kc;
        }
        const int par = round++ & 1;
        red[par][warp][lane] = lane_column_sum(x, lane);
        __syncthreads();
        const float bk = bt * kc;
        float cs[32];
        col_sums(par, cs);
#pragma unroll
        for (int j = 0; j < 32; ++j) S[j] = fmaf(bk, vv[j] - cs[j], S[j]);
        if (u_out && c < 32) {
            const float vj = to_f32(v[((size_t)t * p.H + h) * p.Dv + col0 + c]);
            u_out[c] = vj - col_sum(par, c);
        }
    };

    // ---------------------------------------------- pass A: checkpoints every kBwStep tokens
    float S[32];
    {
        const float *src = p.S0 ? p.S0 + (((size_t)n * p.H + h) * DK + c) * p.Dv + col0 : nullptr;
        if (src) load32(src, S);
        else
#pragma unroll
            for (int j = 0; j < 32; ++j) S[j] = 0.f;
    }
    for (int j = 0; j < nc; ++j) {
        store32(ckpt_row(j), S);
        const int c0 = t0 + j * kBwStep, c1 = min(t1, c0 + kBwStep);
        for (int t = c0; t < c1; ++t) forward_token(t, S, nullptr);
    }

    // ---------------------------------------------- pass B: reverse, step by step
    float G[32];
    {
        const float *src = p.dSf ? p.dSf + (((size_t)n * p.H + h) * DK + c) * p.Dv + col0 : nullptr;
        if (src) load32(src, G);
        else
#pragma unroll
            for (int j = 0; j < 32; ++j) G[j] = 0.f;
    }
    for (int j = nc - 1; j >= 0; --j) {
        const int c0 = t0 + j * kBwStep, L = min(kBwStep, t1 - c0);
        load32(ckpt_row(j), S);
        for (int i = 0; i < L; ++i) {   // states S_{t-1} and u of the chunk's tokens
            store32(scr + ((size_t)i * DK + c) * kBwVs, S);
            forward_token(c0 + i, S, scr_u + i * kBwVs);
        }
        __syncthreads();   // u of every token written before any thread reads it
        for (int i = L - 1; i >= 0; --i) {
            const int t = c0 + i;
            const size_t rk = ((size_t)t * p.H + h) * DK + c;
            if (i > 0) {   // the next (earlier) token's inputs, state row and u
                prefetch_token(t - 1, true);
                prefetch_l1(scr + ((size_t)(i - 1) * DK + c) * kBwVs);
                if (c == 0) prefetch_l1(scr_u + (i - 1) * kBwVs);
            }
            const float qc = to_f32(q[rk]), kc = to_f32(k[rk]), ac = expf(to_f32(la[rk]));
            const float bt = to_f32(beta[(size_t)t * p.H + h]);
            float Sp[32], x[32], u[32];
            load32(scr + ((size_t)i * DK + c) * kBwVs, Sp);
            load32(dout + ((size_t)t * p.H + h) * p.Dv + col0, x);   // do_t
            load32(scr_u + i * kBwVs, u);
            // 4'. dq_t = S_t do_t;  G += q_t do_t^T
            float dq_c = 0.f;
#pragma unroll
            for (int jj = 0; jj < 32; ++jj) {
                dq_c = fmaf(S[jj], x[jj], dq_c);
                G[jj] = fmaf(qc, x[jj], G[jj]);
            }
            // 3'. du = beta G^T k (column sums), k^T G u (dbeta)
            float ge = 0.f;
#pragma unroll
            for (int jj = 0; jj < 32; ++jj) {
                ge = fmaf(G[jj], u[jj], ge);
                x[jj] = G[jj] * kc;
            }
            const int par = round++ & 1;
            red[par][warp][lane] = lane_column_sum(x, lane);
            const float kb = warp_sum(kc * ge);
            if (lane == 0) redb[par][warp] = kb;
            __syncthreads();
            float du[32];
            col_sums(par, du);
#pragma unroll
            for (int jj = 0; jj < 32; ++jj) du[jj] *= bt;
            if (c < 32) p.dv[((size_t)t * p.H + h) * p.Dv + col0 + c] = bt * col_sum(par, c);
            if (c == 0) {
                float db = 0.f;
#pragma unroll
                for (int w = 0; w < NW; ++w) db += redb[par][w];
                part_db[(size_t)t * p.H + h] = db;
            }
            // 2'. dk_t = beta G u - P du,  dP = G - k du^T
            // 1'. dlog_alpha_t = alpha rowsum(dP * S_{t-1}),  G = Diag(alpha) dP
            float pdu = 0.f, dps = 0.f;
#pragma unroll
            for (int jj = 0; jj < 32; ++jj) {
                pdu = fmaf(ac * Sp[jj], du[jj], pdu);
                const float dP = fmaf(-kc, du[jj], G[jj]);
                dps = fmaf(dP, Sp[jj], dps);
                G[jj] = ac * dP;
                S[jj] = Sp[jj];
            }
            part_dq[rk] = dq_c;
            part_dk[rk] = fmaf(bt, ge, -pdu);
            part_dla[rk] = ac * dps;
        }
    }
    if (p.dS0) store32(p.dS0 + (((size_t)n * p.H + h) * DK + c) * p.Dv + col0, G);
}

// dq, dk, dlog_alpha and dbeta = the slices' partial sums added in slice
// order.  Four float elements per thread (every region is a multiple of 4
// floats long: T H DK with DK in {64, 128}; T H padded in the workspace).
__global__ void __launch_bounds__(256)
slice_sum_kernel(const float *__restrict__ part, size_t part_stride, int n_slices, size_t thd,
                 size_t th, float *dq, float *dk, float *dla, float *dbeta) {
    const size_t n4 = (3 * thd + th + 3) / 4;
    for (size_t i4 = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i4 < n4;
         i4 += (size_t)gridDim.x * blockDim.x) {
        const size_t i = 4 * i4;
        float4 acc = reinterpret_cast<const float4 *>(part + i)[0];
        for (int sl = 1; sl < n_slices; ++sl) {
            const float4 x = reinterpret_cast<const float4 *>(part + (size_t)sl * part_stride + i)[0];
            acc.x += x.x; acc.y += x.y; acc.z += x.z; acc.w += x.w;
        }
        if (i < 3 * thd) {
            float *dst = i < thd ? dq + i : i < 2 * thd ? dk + (i - thd) : dla + (i - 2 * thd);
            *reinterpret_cast<float4 *>(dst) = acc;
        } else {
            // dbeta is not padded: store only its T H elements
            const size_t j = i - 3 * thd;
            const float v4[4] = {acc.x, acc.y, acc.z, acc.w};
            for (int e = 0; e < 4 && j + e < th; ++e) dbeta[j + e] = v4[e];
        }
    }
}

template <typename TIO, typename TG, int DK>
cudaError_t launch_bw(const BwParams &bp, cudaStream_t s) {
    const unsigned grid = (unsigned)bp.N * bp.H * (bp.Dv / kBwVs);
    backward_kernel<TIO, TG, DK><<<grid, DK, 0, s>>>(bp);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || bp.T == 0) return e;
    const size_t thd = (size_t)bp.T * bp.H * DK, th = (size_t)bp.T * bp.H;
    const size_t n4 = (3 * thd + th + 3) / 4;
    const unsigned blocks = (unsigned)((n4 + 255) / 256 < 148 * 8 ? (n4 + 255) / 256 : 148 * 8);
    slice_sum_kernel<<<blocks, 256, 0, s>>>(bp.part, bp.part_stride, bp.Dv / kBwVs, thd, th, bp.dq,
                                            bp.dk, bp.dla, bp.dbeta);
    return cudaGetLastError();
}

template <typename TIO, typename TG>
cudaError_t launch_bw_dk(const BwParams &bp, int Dk, cudaStream_t s) {
    return Dk == 64 ? launch_bw<TIO, TG, 64>(bp, s) : launch_bw<TIO, TG, 128>(bp, s);
}

}  // namespace

cudaError_t launch_backward(const BackwardArgs &a, cudaStream_t s) {
    // with no tokens at all the chains still pass dS_final (or zero) on to dS0
    if (a.N == 0) return cudaSuccess;
    BwParams bp;
    bp.q = a.q; bp.k = a.k; bp.v = a.v; bp.la = a.log_alpha; bp.beta = a.beta;
    bp.d_out = a.d_out; bp.S0 = a.S0; bp.dSf = a.dS_final;
    bp.cu = a.cu_seqlens; bp.order = a.order; bp.chunk_off = a.chunk_off;
    bp.dq = a.dq; bp.dk = a.dk; bp.dv = a.dv; bp.dla = a.dla; bp.dbeta = a.dbeta;
    bp.dS0 = a.dS0; bp.ckpt = a.ckpt; bp.scratch = a.scratch;
    bp.part = a.part; bp.part_stride = a.part_stride;
    bp.ckpt_steps = (long long)a.ckpt_steps; bp.status = a.status;
    bp.N = a.N; bp.T = a.T; bp.H = a.H; bp.Dv = a.Dv;
    const bool io_bf16 = a.io_dtype == KDA_BF16, g_bf16 = a.gate_dtype == KDA_BF16;
    if (io_bf16 && g_bf16) return launch_bw_dk<__nv_bfloat16, __nv_bfloat16>(bp, a.Dk, s);
    if (io_bf16) return launch_bw_dk<__nv_bfloat16, float>(bp, a.Dk, s);
    if (g_bf16) return launch_bw_dk<float, __nv_bfloat16>(bp, a.Dk, s);
    return launch_bw_dk<float, float>(bp, a.Dk, s);
}

}  // namespace kda
