// kda_decode.cu -- recurrent KDA tokens for N independent sequences: one
// token per call (state updated in place), or several consecutive tokens per
// sequence with the state read once and the state after every token kept
// (for a verify step of speculative decoding that may roll back).
//
// Per (sequence, head) the step of the page "Kimi K3: Open Frontier
// Intelligence and Implementation Framework" (section "Hybrid Attention
// Mechanism", KDA bullet) is, with a = exp(log_alpha):
//     y_k = (Diag(a) S)^T k,  y_q = (Diag(a) S)^T q        (one read of S)
//     u   = beta (v - y_k)
//     o   = y_q + (q . k) u                                 (= S_new^T q)
//     S   <- Diag(a) S + k u^T                              (one write of S)
// which is S_new = (I - beta k k^T) Diag(a) S + beta k v^T written so that
// the fp32 state is streamed from HBM exactly once in each direction.
//
// Layout: S [N, H, Dk, Dv] fp32 with Dv contiguous.  A CTA of 128 threads
// owns one (sequence, head, 64-column slice of Dv): thread (rg, cg) holds
// rows rg*Dk/8 .. +Dk/8 of four adjacent columns 4cg..4cg+3 in registers
// (one 16-byte load and store per row), so the state never touches shared
// memory; the two column sums are reduced across the 8 row groups through
// shared memory.  Columns are separable, so slices need no communication.
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kThreads = 128;
constexpr int kCols = 64;   // Dv columns per CTA
constexpr int kRowGroups = 8;

template <typename TIO, typename TG, int DK>
__global__ void __launch_bounds__(kThreads)
decode_kernel(const TIO *__restrict__ q, const TIO *__restrict__ k, const TIO *__restrict__ v,
              const TG *__restrict__ la, const TG *__restrict__ beta, float *__restrict__ S,
              float *__restrict__ S_tokens, TIO *__restrict__ out, int H, int Dv, int n_tokens) {
    constexpr int RPT = DK / kRowGroups;  // rows per thread
    __shared__ float s_a[DK], s_ka[DK], s_qa[DK], s_k[DK];
    __shared__ float s_red[2][kRowGroups][kCols];
    __shared__ float s_qk;

    const int slices = Dv / kCols;
    const int nh = blockIdx.x / slices;        // n * H + h
    const int n = nh / H, h = nh % H;
    const int col0 = (blockIdx.x % slices) * kCols;
    const int tid = threadIdx.x;
    const int cg = tid % 16, rg = tid / 16;

    // Issue the state loads first: they are the only long-latency traffic.
    float *Sp = S + (size_t)nh * DK * Dv + col0 + cg * 4;
    float4 st[RPT];
#pragma unroll
    for (int i = 0; i < RPT; ++i)
        st[i] = *reinterpret_cast<const float4 *>(Sp + (size_t)(rg * RPT + i) * Dv);

    // Tokens of one sequence are consecutive rows of the token-major inputs;
    // the state stays in registers from one token to the next.
    for (int t = 0; t < n_tokens; ++t) {
        const size_t row = ((size_t)n * n_tokens + t) * H + h;   // (n, t, h)
        const size_t vbase = row * DK;
        if (t > 0) __syncthreads();   // everyone is done with the previous token's vectors
        for (int c = tid; c < DK; c += kThreads) {
            const float a = expf(to_f32(la[vbase + c]));
            const float kc = to_f32(k[vbase + c]);
            s_a[c] = a;
            s_k[c] = kc;
            s_ka[c] = kc * a;
            s_qa[c] = to_f32(q[vbase + c]) * a;
        }
        if (tid < 32) {
            float p = 0.f;
            for (int c = tid; c < DK; c += 32) p = fmaf(to_f32(q[vbase + c]), to_f32(k[vbase + c]), p);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) p += __shfl_xor_sync(0xffffffffu, p, o);
            if (tid == 0) s_qk = p;
        }
        __syncthreads();

        float yk[4] = {0.f, 0.f, 0.f, 0.f}, yq[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
            const int c = rg * RPT + i;
            const float ka = s_ka[c], qa = s_qa[c];
            yk[0] = fmaf(ka, st[i].x, yk[0]); yq[0] = fmaf(qa, st[i].x, yq[0]);
            yk[1] = fmaf(ka, st[i].y, yk[1]); yq[1] = fmaf(qa, st[i].y, yq[1]);
            yk[2] = fmaf(ka, st[i].z, yk[2]); yq[2] = fmaf(qa, st[i].z, yq[2]);
            yk[3] = fmaf(ka, st[i].w, yk[3]); yq[3] = fmaf(qa, st[i].w, yq[3]);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            s_red[0][rg][cg * 4 + j] = yk[j];
            s_red[1][rg][cg * 4 + j] = yq[j];
        }
        __syncthreads();

        const float b = to_f32(beta[row]);
        const float qk = s_qk;
        float u[4], o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float sk = 0.f, sq = 0.f;
#pragma unroll
            for (int g = 0; g < kRowGroups; ++g) {
                sk += s_red[0][g][cg * 4 + j];
                sq += s_red[1][g][cg * 4 + j];
            }
            const float vj = to_f32(v[row * Dv + col0 + cg * 4 + j]);
            u[j] = b * (vj - sk);
            o[j] = fmaf(qk, u[j], sq);
        }

        // the state after this token: in place for a single step, else into
        // its own slot of S_tokens [N, n_tokens, H, Dk, Dv]
        float *Sw = S_tokens ? S_tokens + row * DK * Dv + col0 + cg * 4 : Sp;
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
            const int c = rg * RPT + i;
            const float a = s_a[c], kc = s_k[c];
            float4 w;
            w.x = fmaf(a, st[i].x, kc * u[0]);
            w.y = fmaf(a, st[i].y, kc * u[1]);
            w.z = fmaf(a, st[i].z, kc * u[2]);
            w.w = fmaf(a, st[i].w, kc * u[3]);
            st[i] = w;
            if (S_tokens || t == n_tokens - 1)
                *reinterpret_cast<float4 *>(Sw + (size_t)c * Dv) = w;
        }
        if (rg == 0) {
            TIO *op = out + row * Dv + col0 + cg * 4;
#pragma unroll
            for (int j = 0; j < 4; ++j) op[j] = from_f32<TIO>(o[j]);
        }
    }
}

template <typename TIO, typename TG, int DK>
cudaError_t launch_typed(const DecodeArgs &a, cudaStream_t s) {
    const unsigned grid = (unsigned)((size_t)a.N * a.H * (a.Dv / kCols));
    decode_kernel<TIO, TG, DK><<<grid, kThreads, 0, s>>>(
        (const TIO *)a.q, (const TIO *)a.k, (const TIO *)a.v, (const TG *)a.log_alpha,
        (const TG *)a.beta, a.S, a.S_tokens, (TIO *)a.out, a.H, a.Dv, a.n_tokens);
    return cudaGetLastError();
}

template <typename TIO, typename TG>
cudaError_t launch_dk(const DecodeArgs &a, cudaStream_t s) {
    return a.Dk == 64 ? launch_typed<TIO, TG, 64>(a, s) : launch_typed<TIO, TG, 128>(a, s);
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t s) {
    const bool io16 = a.io_dtype == KDA_BF16, g16 = a.gate_dtype == KDA_BF16;
    if (io16 && g16) return launch_dk<__nv_bfloat16, __nv_bfloat16>(a, s);
    if (io16) return launch_dk<__nv_bfloat16, float>(a, s);
    if (g16) return launch_dk<float, __nv_bfloat16>(a, s);
    return launch_dk<float, float>(a, s);
}

}  // namespace kda
