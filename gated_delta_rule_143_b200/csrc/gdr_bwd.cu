// gdr_bwd.cu -- gradients of the gated delta-rule forward (dq, dk, dv, dg, dbeta, dS0) on the CUDA
// cores in fp32.
//
// The forward is the token recurrence of "Linear Attention & DeltaNet" (How it works, items 3-4) with
// the decay of "linear attention and its gated descendants" (Gated DeltaNet, Kimi Delta Attention).
// Row j of the state (s_j in R^{d_k}) evolves on its own given k, q, beta and alpha = exp(g):
//
//   s_bar = s (.) alpha ;  p = s_bar . k ;  delta = beta (v_j - p) ;  s' = s_bar + delta k ;
//   o_j = scale (s' . q)
//
// and its reverse-mode gradient, with ds the gradient of the row after the token, is
//
//   ds'    = ds + scale do_j q            dq += scale do_j s'
//   ddelta = ds' . k                      dk += delta ds'
//   dbeta += ddelta (v_j - p)             dv_j = beta ddelta
//   ds_bar = ds' - beta ddelta k          dk += -beta ddelta s_bar
//   ds     = ds_bar (.) alpha             dg += ds_bar (.) s_bar
//
// dq, dk, dbeta and dg sum over the d_v rows (and over the key channels for the scalar gate).
//
// Two kernels, one CTA per (b, h), 16 warps with d_v / 16 rows each (the rows in registers; lane l
// holds key channels l + 32 i):
//  1. history: runs the recurrence forward and stores the state before every token in the workspace
//     (T x d_v x d_k fp32 per head), so that the reverse sweep needs no recomputation;
//  2. reverse: walks the tokens from the last to the first with ds in registers, reads the stored
//     state of each token, and reduces the row sums across the warps in shared memory (one barrier
//     per token, double-buffered). dv is per row and goes straight out.
// Both are bound by HBM (the history is written once and read once); this form trades memory for
// simplicity: the workspace is B * H * T * d_v * d_k * 4 bytes.
#include "gdr_internal.cuh"

namespace gdr {
namespace {

constexpr int kBwdWarps = 16;
constexpr int kBwdThreads = kBwdWarps * 32;

__device__ __forceinline__ float bwd_warp_sum(float x) {
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
    return x;
}

struct BwdArgs {
    const void* q;
    const void* k;
    const void* v;
    const float* g;
    const float* beta;
    const float* S0;
    const void* dO;
    const float* dST;
    float* dq;
    float* dk;
    float* dv;
    float* dg;
    float* dbeta;
    float* dS0;
    float* hist;  // [B*H][T][d_v][d_k]
    int T, H, dv_;
    float scale;
};

// Decay factors of token `tok` for this lane's channels.
template <int MODE, int NL>
__device__ __forceinline__ void load_alpha(const float* g, size_t tok, int lane, float (&a)[NL]) {
    if (MODE == GDR_DECAY_CHANNEL) {
#pragma unroll
        for (int i = 0; i < NL; ++i) a[i] = expf(g[tok * (NL * 32) + lane + 32 * i]);
    } else {
        const float x = MODE == GDR_DECAY_SCALAR ? expf(g[tok]) : 1.f;
#pragma unroll
        for (int i = 0; i < NL; ++i) a[i] = x;
    }
}

template <typename Tin, int MODE, int DK, int RPW>
__global__ void __launch_bounds__(kBwdThreads)
bwd_history_kernel(BwdArgs A) {
    constexpr int NL = DK / 32;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const size_t bh = blockIdx.x;
    const int h = (int)(bh % A.H), b = (int)(bh / A.H);
    const int dv = A.dv_, T = A.T;
    const Tin* k = static_cast<const Tin*>(A.k);
    const Tin* v = static_cast<const Tin*>(A.v);
    float s[RPW][NL];
#pragma unroll
    for (int r = 0; r < RPW; ++r) {
        const int j = warp * RPW + r;
#pragma unroll
        for (int i = 0; i < NL; ++i)
            s[r][i] = A.S0 != nullptr ? A.S0[(bh * dv + j) * DK + lane + 32 * i] : 0.f;
    }
    for (int t = 0; t < T; ++t) {
        const size_t tok = ((size_t)b * T + t) * A.H + h;
        float kk[NL], a[NL];
#pragma unroll
        for (int i = 0; i < NL; ++i) kk[i] = load_f32(k + tok * DK + lane + 32 * i);
        load_alpha<MODE, NL>(A.g, tok, lane, a);
        const float bt = A.beta[tok];
        float* hrow = A.hist + ((bh * T + t) * dv) * DK;
#pragma unroll
        for (int r = 0; r < RPW; ++r) {
            const int j = warp * RPW + r;
            float p = 0.f;
#pragma unroll
            for (int i = 0; i < NL; ++i) {
                hrow[(size_t)j * DK + lane + 32 * i] = s[r][i];
                s[r][i] *= a[i];
                p = fmaf(s[r][i], kk[i], p);
            }
            p = bwd_warp_sum(p);
            const float d = bt * (load_f32(v + tok * dv + j) - p);
#pragma unroll
            for (int i = 0; i < NL; ++i) s[r][i] = fmaf(d, kk[i], s[r][i]);
        }
    }
}

template <typename Tin, int MODE, int DK, int RPW>
__global__ void __launch_bounds__(kBwdThreads)
bwd_reverse_kernel(BwdArgs A) {
    constexpr int NL = DK / 32;
    // per buffer: [warp][dq | dk | dg][DK] partial sums, then [warp] dbeta and scalar-gate dg
    extern __shared__ float bwd_smem[];
    auto red = reinterpret_cast<float(*)[kBwdWarps][3][DK]>(bwd_smem);
    auto redb = reinterpret_cast<float(*)[kBwdWarps][2]>(bwd_smem + 2 * kBwdWarps * 3 * DK);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const size_t bh = blockIdx.x;
    const int h = (int)(bh % A.H), b = (int)(bh / A.H);
    const int dv = A.dv_, T = A.T;
    const Tin* q = static_cast<const Tin*>(A.q);
    const Tin* k = static_cast<const Tin*>(A.k);
    const Tin* v = static_cast<const Tin*>(A.v);
    const Tin* dO = static_cast<const Tin*>(A.dO);
    const float sc = A.scale;
    float ds[RPW][NL];
#pragma unroll
    for (int r = 0; r < RPW; ++r) {
        const int j = warp * RPW + r;
#pragma unroll
        for (int i = 0; i < NL; ++i) ds[r][i] = A.dST != nullptr ? A.dST[(bh * dv + j) * DK + lane + 32 * i] : 0.f;
    }
    for (int t = T - 1; t >= 0; --t) {
        const int buf = t & 1;
        const size_t tok = ((size_t)b * T + t) * A.H + h;
        float kk[NL], qq[NL], a[NL];
#pragma unroll
        for (int i = 0; i < NL; ++i) {
            kk[i] = load_f32(k + tok * DK + lane + 32 * i);
            qq[i] = load_f32(q + tok * DK + lane + 32 * i);
        }
        load_alpha<MODE, NL>(A.g, tok, lane, a);
        const float bt = A.beta[tok];
        const float* hrow = A.hist + ((bh * T + t) * dv) * DK;
        float gq[NL], gk[NL], gg[NL], gb = 0.f;
#pragma unroll
        for (int i = 0; i < NL; ++i) gq[i] = gk[i] = gg[i] = 0.f;
#pragma unroll
        for (int r = 0; r < RPW; ++r) {
            const int j = warp * RPW + r;
            float sb[NL], p = 0.f;
#pragma unroll
            for (int i = 0; i < NL; ++i) {
                sb[i] = hrow[(size_t)j * DK + lane + 32 * i] * a[i];
                p = fmaf(sb[i], kk[i], p);
            }
            p = bwd_warp_sum(p);
            const float vj = load_f32(v + tok * dv + j);
            const float doj = sc * load_f32(dO + tok * dv + j);
            const float delta = bt * (vj - p);
            float dsp[NL], dd = 0.f;
#pragma unroll
            for (int i = 0; i < NL; ++i) {
                dsp[i] = fmaf(doj, qq[i], ds[r][i]);
                gq[i] = fmaf(doj, fmaf(delta, kk[i], sb[i]), gq[i]);
                gk[i] = fmaf(delta, dsp[i], gk[i]);
                dd = fmaf(dsp[i], kk[i], dd);
            }
            dd = bwd_warp_sum(dd);
            gb = fmaf(dd, vj - p, gb);
            if (lane == 0) A.dv[tok * dv + j] = bt * dd;
            const float dp = -bt * dd;
#pragma unroll
            for (int i = 0; i < NL; ++i) {
                const float dsb = fmaf(dp, kk[i], dsp[i]);
                gk[i] = fmaf(dp, sb[i], gk[i]);
                gg[i] = fmaf(dsb, sb[i], gg[i]);
                ds[r][i] = dsb * a[i];
            }
        }
        // row sums of this warp into the buffer of token t; one barrier, then the sums across the
        // warps (the other buffer is free: its readers finished before this barrier)
#pragma unroll
        for (int i = 0; i < NL; ++i) {
            red[buf][warp][0][lane + 32 * i] = gq[i];
            red[buf][warp][1][lane + 32 * i] = gk[i];
            red[buf][warp][2][lane + 32 * i] = gg[i];
        }
        if (MODE == GDR_DECAY_SCALAR) {
            float x = 0.f;
#pragma unroll
            for (int i = 0; i < NL; ++i) x += gg[i];
            x = bwd_warp_sum(x);
            if (lane == 0) redb[buf][warp][1] = x;
        }
        if (lane == 0) redb[buf][warp][0] = gb;
        __syncthreads();
        const int tid = threadIdx.x;
        const int nsum = MODE == GDR_DECAY_CHANNEL ? 3 * DK : 2 * DK;
        if (tid < nsum) {
            const int which = tid / DK, c = tid % DK;
            float x = 0.f;
#pragma unroll
            for (int w = 0; w < kBwdWarps; ++w) x += red[buf][w][which][c];
            float* dst = which == 0 ? A.dq : (which == 1 ? A.dk : A.dg);
            dst[tok * DK + c] = x;
        } else if (tid == nsum || tid == nsum + 1) {
            const int which = tid - nsum;  // 0: dbeta, 1: scalar-gate dg
            if (which == 0 || MODE == GDR_DECAY_SCALAR) {
                float x = 0.f;
#pragma unroll
                for (int w = 0; w < kBwdWarps; ++w) x += redb[buf][w][which];
                if (which == 0) A.dbeta[tok] = x;
                else A.dg[tok] = x;
            }
        }
    }
    if (A.dS0 != nullptr) {
#pragma unroll
        for (int r = 0; r < RPW; ++r) {
            const int j = warp * RPW + r;
#pragma unroll
            for (int i = 0; i < NL; ++i) A.dS0[(bh * dv + j) * DK + lane + 32 * i] = ds[r][i];
        }
    }
}

template <typename Tin, int MODE, int DK, int RPW>
cudaError_t launch_bwd_typed(const BwdArgs& a, int BH, cudaStream_t stream) {
    bwd_history_kernel<Tin, MODE, DK, RPW><<<BH, kBwdThreads, 0, stream>>>(a);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    auto kern = bwd_reverse_kernel<Tin, MODE, DK, RPW>;
    const size_t smem = (size_t)2 * kBwdWarps * (3 * DK + 2) * sizeof(float);
    if ((err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
        return err;
    kern<<<BH, kBwdThreads, smem, stream>>>(a);
    return cudaGetLastError();
}

template <typename Tin, int MODE, int DK>
cudaError_t launch_bwd_dv(const BwdArgs& a, int BH, cudaStream_t stream) {
    switch (a.dv_) {
        case 32: return launch_bwd_typed<Tin, MODE, DK, 2>(a, BH, stream);
        case 64: return launch_bwd_typed<Tin, MODE, DK, 4>(a, BH, stream);
        case 128: return launch_bwd_typed<Tin, MODE, DK, 8>(a, BH, stream);
        default: return cudaErrorInvalidValue;
    }
}

template <typename Tin, int MODE>
cudaError_t launch_bwd_dk(const BwdArgs& a, int dk, int BH, cudaStream_t stream) {
    switch (dk) {
        case 32: return launch_bwd_dv<Tin, MODE, 32>(a, BH, stream);
        case 64: return launch_bwd_dv<Tin, MODE, 64>(a, BH, stream);
        case 128: return launch_bwd_dv<Tin, MODE, 128>(a, BH, stream);
        default: return cudaErrorInvalidValue;
    }
}

template <typename Tin>
cudaError_t launch_bwd_mode(const BwdArgs& a, int mode, int dk, int BH, cudaStream_t stream) {
    switch (mode) {
        case GDR_DECAY_NONE: return launch_bwd_dk<Tin, GDR_DECAY_NONE>(a, dk, BH, stream);
        case GDR_DECAY_SCALAR: return launch_bwd_dk<Tin, GDR_DECAY_SCALAR>(a, dk, BH, stream);
        case GDR_DECAY_CHANNEL: return launch_bwd_dk<Tin, GDR_DECAY_CHANNEL>(a, dk, BH, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

bool bwd_supported(int dk, int dv) {
    return (dk == 32 || dk == 64 || dk == 128) && (dv == 32 || dv == 64 || dv == 128);
}

size_t bwd_workspace_bytes(int B, int T, int H, int dk, int dv) {
    return (size_t)B * H * T * dv * dk * sizeof(float);
}

cudaError_t launch_bwd(const BwdProblem& p, cudaStream_t stream) {
    BwdArgs a{p.q,  p.k,  p.v,  p.g,     p.beta, p.S0, p.dO, p.dST, p.dq, p.dk, p.dv,
              p.dg, p.dbeta, p.dS0, static_cast<float*>(p.workspace), p.T, p.H, p.dv_dim, p.scale};
    const int BH = p.B * p.H;
    if (p.dtype == GDR_BF16) return launch_bwd_mode<__nv_bfloat16>(a, p.mode, p.dk_dim, BH, stream);
    return launch_bwd_mode<float>(a, p.mode, p.dk_dim, BH, stream);
}

}  // namespace gdr
