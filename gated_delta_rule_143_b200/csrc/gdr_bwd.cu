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
// Two kernels, 4 warps per CTA, d_v / 8 CTAs per (b, h) with two state rows a warp (the history
// kernel: d_v / 4 CTAs, one row a warp) (the rows in registers;
// lane l holds key channels l + 32 i), each token's inputs loaded one token ahead of their use:
//  1. history: runs the recurrence forward and stores the state before every token in the workspace
//     (T x d_v x d_k fp32 per head), so that the reverse sweep needs no recomputation;
//  2. reverse: walks the tokens from the last to the first with ds in registers, reads the stored
//     state of each token from a 3-stage ring in shared memory filled by bulk copies three tokens
//     ahead (mbarrier waits bounded like the tensor-core kernels'), and reduces the row sums across the warps in shared memory (one barrier
//     per token, double-buffered), then across the head's CTAs with vector atomics into zeroed
//     outputs (plain stores when one CTA holds the head). dv is per row and goes straight out.
// Both are bound by HBM (the history is written once and read once); this form trades memory for
// simplicity: the workspace is B * H * T * d_v * d_k * 4 bytes.
#include "gdr_sm100.cuh"

namespace gdr {
namespace {

using namespace sm100;

constexpr int kBwdWarps = 4;  // small CTAs: 20 % faster reverse sweep than 16 warps (more CTAs per SM)
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
    int* status;
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

// Rows of the state per warp and per CTA: a head's d_v rows are spread over d_v / 8 CTAs (more SMs
// at work); the row sums of dq, dk, dg and dbeta then meet in global memory (vector atomics) unless
// one CTA holds the whole head.
constexpr int kBwdRowsPerWarp = 2;
constexpr int kBwdRowsPerCta = kBwdWarps * kBwdRowsPerWarp;  // 8

constexpr int kBwdStages = 3;  // reverse sweep: stored state rows in flight, one CTA-slice per token
// The history kernel's warps take one row each: twice the warps (and stores) in flight of two rows a
// warp, for a sweep that waits on memory.
constexpr int kHistRowsPerWarp = 1;
constexpr int kHistRowsPerCta = kBwdWarps * kHistRowsPerWarp;

// The inputs of one token that a warp needs, loaded one token ahead of their use.
template <int NL>
struct BwdToken {
    float kk[NL], qq[NL], a[NL], bt;
    float vj[kBwdRowsPerWarp], doj[kBwdRowsPerWarp];
};

template <typename Tin, int MODE, int DK>
__global__ void __launch_bounds__(kBwdThreads)
bwd_history_kernel(BwdArgs A) {
    constexpr int NL = DK / 32, R = kHistRowsPerWarp;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const size_t bh = blockIdx.y;
    const int h = (int)(bh % A.H), b = (int)(bh / A.H);
    const int dv = A.dv_, T = A.T;
    const int j0 = blockIdx.x * kHistRowsPerCta + warp * R;  // this warp's first state row
    const Tin* k = static_cast<const Tin*>(A.k);
    const Tin* v = static_cast<const Tin*>(A.v);
    auto load = [&](int t, BwdToken<NL>& x) {
        const size_t tok = ((size_t)b * T + t) * A.H + h;
#pragma unroll
        for (int i = 0; i < NL; ++i) x.kk[i] = load_f32(k + tok * DK + lane + 32 * i);
        load_alpha<MODE, NL>(A.g, tok, lane, x.a);
        x.bt = A.beta[tok];
#pragma unroll
        for (int r = 0; r < R; ++r) x.vj[r] = load_f32(v + tok * dv + j0 + r);
    };
    float s[R][NL];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int i = 0; i < NL; ++i)
            s[r][i] = A.S0 != nullptr ? A.S0[(bh * dv + j0 + r) * DK + lane + 32 * i] : 0.f;
    BwdToken<NL> cur, nxt;
    load(0, cur);
    for (int t = 0; t < T; ++t) {
        if (t + 1 < T) load(t + 1, nxt);  // in flight while this token is computed
        float* hrow = A.hist + ((bh * T + t) * dv) * DK;
#pragma unroll
        for (int r = 0; r < R; ++r) {
            float p = 0.f;
#pragma unroll
            for (int i = 0; i < NL; ++i) {
                hrow[(size_t)(j0 + r) * DK + lane + 32 * i] = s[r][i];
                s[r][i] *= cur.a[i];
                p = fmaf(s[r][i], cur.kk[i], p);
            }
            p = bwd_warp_sum(p);
            const float d = cur.bt * (cur.vj[r] - p);
#pragma unroll
            for (int i = 0; i < NL; ++i) s[r][i] = fmaf(d, cur.kk[i], s[r][i]);
        }
        cur = nxt;
    }
}

template <typename Tin, int MODE, int DK>
__global__ void __launch_bounds__(kBwdThreads)
bwd_reverse_kernel(BwdArgs A) {
    constexpr int NL = DK / 32, R = kBwdRowsPerWarp;
    // per buffer: [warp][dq | dk | dg][DK] partial sums, then [warp] dbeta and scalar-gate dg; then
    // the ring of stored state rows: the CTA's 8 rows of one token per stage, brought in by bulk
    // copies kBwdStages tokens ahead
    extern __shared__ float bwd_smem[];
    auto red = reinterpret_cast<float(*)[kBwdWarps][3][DK]>(bwd_smem);
    auto redb = reinterpret_cast<float(*)[kBwdWarps][2]>(bwd_smem + 2 * kBwdWarps * 3 * DK);
    float* ring = bwd_smem + 2 * kBwdWarps * (3 * DK + 2);
    constexpr uint32_t kStageFloats = kBwdRowsPerCta * DK, kStageBytes = kStageFloats * 4;
    __shared__ uint64_t full[kBwdStages];
    __shared__ int abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const size_t bh = blockIdx.y;
    const int h = (int)(bh % A.H), b = (int)(bh / A.H);
    const int dv = A.dv_, T = A.T;
    const int j0 = blockIdx.x * kBwdRowsPerCta + warp * R;
    const bool whole_head = gridDim.x == 1;  // plain stores; otherwise the CTAs of a head add up
    if (threadIdx.x == 0) {
        for (int st = 0; st < kBwdStages; ++st) mbar_init(&full[st], 1);
        fence_mbar_init();
        abort_flag = 0;
    }
    __syncthreads();
    // u-th token of the sweep (t = T - 1 - u) into stage u % kBwdStages
    auto issue = [&](int u) {
        const int st = u % kBwdStages;
        mbar_arrive_expect_tx(&full[st], kStageBytes);
        bulk_g2s(ring + st * kStageFloats,
                 A.hist + ((bh * T + (T - 1 - u)) * dv + (size_t)blockIdx.x * kBwdRowsPerCta) * DK, kStageBytes,
                 &full[st]);
    };
    if (threadIdx.x == 0)
        for (int u = 0; u < kBwdStages && u < T; ++u) issue(u);
    const Tin* q = static_cast<const Tin*>(A.q);
    const Tin* k = static_cast<const Tin*>(A.k);
    const Tin* v = static_cast<const Tin*>(A.v);
    const Tin* dO = static_cast<const Tin*>(A.dO);
    const float sc = A.scale;
    auto load = [&](int t, BwdToken<NL>& x) {
        const size_t tok = ((size_t)b * T + t) * A.H + h;
#pragma unroll
        for (int i = 0; i < NL; ++i) {
            x.kk[i] = load_f32(k + tok * DK + lane + 32 * i);
            x.qq[i] = load_f32(q + tok * DK + lane + 32 * i);
        }
        load_alpha<MODE, NL>(A.g, tok, lane, x.a);
        x.bt = A.beta[tok];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            x.vj[r] = load_f32(v + tok * dv + j0 + r);
            x.doj[r] = sc * load_f32(dO + tok * dv + j0 + r);
        }
    };
    float ds[R][NL];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int i = 0; i < NL; ++i)
            ds[r][i] = A.dST != nullptr ? A.dST[(bh * dv + j0 + r) * DK + lane + 32 * i] : 0.f;
    BwdToken<NL> cur, nxt;
    load(T - 1, cur);
    bool ok = true;  // false once a wait has expired (the status word then says so)
    for (int t = T - 1, u = 0; t >= 0; --t, ++u) {
        if (t > 0) load(t - 1, nxt);  // the next token's inputs, in flight
        const int buf = t & 1, st = u % kBwdStages;
        ok = ok && mbar_wait_abort(&full[st], (uint32_t)(u / kBwdStages) & 1u, A.status, &abort_flag);
        const float* srow = ring + st * kStageFloats + (warp * R) * DK;
        const size_t tok = ((size_t)b * T + t) * A.H + h;
        float gq[NL], gk[NL], gg[NL], gb = 0.f;
#pragma unroll
        for (int i = 0; i < NL; ++i) gq[i] = gk[i] = gg[i] = 0.f;
#pragma unroll
        for (int r = 0; r < R; ++r) {
            float sb[NL], p = 0.f;
#pragma unroll
            for (int i = 0; i < NL; ++i) {
                sb[i] = (ok ? srow[r * DK + lane + 32 * i] : 0.f) * cur.a[i];
                p = fmaf(sb[i], cur.kk[i], p);
            }
            p = bwd_warp_sum(p);
            const float vj = cur.vj[r], doj = cur.doj[r];
            const float delta = cur.bt * (vj - p);
            float dsp[NL], dd = 0.f;
#pragma unroll
            for (int i = 0; i < NL; ++i) {
                dsp[i] = fmaf(doj, cur.qq[i], ds[r][i]);
                gq[i] = fmaf(doj, fmaf(delta, cur.kk[i], sb[i]), gq[i]);
                gk[i] = fmaf(delta, dsp[i], gk[i]);
                dd = fmaf(dsp[i], cur.kk[i], dd);
            }
            dd = bwd_warp_sum(dd);
            gb = fmaf(dd, vj - p, gb);
            if (lane == 0) A.dv[tok * dv + j0 + r] = cur.bt * dd;
            const float dp = -cur.bt * dd;
#pragma unroll
            for (int i = 0; i < NL; ++i) {
                const float dsb = fmaf(dp, cur.kk[i], dsp[i]);
                gk[i] = fmaf(dp, sb[i], gk[i]);
                gg[i] = fmaf(dsb, sb[i], gg[i]);
                ds[r][i] = dsb * cur.a[i];
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
        const int nvec = (MODE == GDR_DECAY_CHANNEL ? 3 : 2) * DK / 4;  // float4 groups of dq | dk | dg
        // one item per float4 group, then dbeta and the scalar gate's dg, strided over the threads
        for (int e = threadIdx.x; e < nvec + 2; e += kBwdThreads) {
            if (e < nvec) {
                const int which = e / (DK / 4), c = 4 * (e % (DK / 4));
                float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int w = 0; w < kBwdWarps; ++w) {
                    const float4 y = *reinterpret_cast<const float4*>(&red[buf][w][which][c]);
                    x.x += y.x;
                    x.y += y.y;
                    x.z += y.z;
                    x.w += y.w;
                }
                float4* dst =
                    reinterpret_cast<float4*>((which == 0 ? A.dq : (which == 1 ? A.dk : A.dg)) + tok * DK + c);
                if (whole_head) *dst = x;
                else atomicAdd(dst, x);
            } else {
                const int which = e - nvec;  // 0: dbeta, 1: scalar-gate dg
                if (which == 0 || MODE == GDR_DECAY_SCALAR) {
                    float x = 0.f;
#pragma unroll
                    for (int w = 0; w < kBwdWarps; ++w) x += redb[buf][w][which];
                    float* dst = which == 0 ? A.dbeta + tok : A.dg + tok;
                    if (whole_head) *dst = x;
                    else atomicAdd(dst, x);
                }
            }
        }
        // every thread has read stage st (the barrier above): it takes the token kBwdStages later
        if (threadIdx.x == 0 && u + kBwdStages < T) issue(u + kBwdStages);
        cur = nxt;
    }
    // after an expired wait, copies may still be in flight: let them land (bounded) before exiting
    if (threadIdx.x == 0 && !ok) {
        for (int st = 0; st < kBwdStages && st < T; ++st) {
            const int last = st + ((T - 1 - st) / kBwdStages) * kBwdStages;  // last token issued to stage st
            mbar_wait(&full[st], (uint32_t)(last / kBwdStages) & 1u, A.status);
        }
    }
    if (A.dS0 != nullptr) {
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int i = 0; i < NL; ++i) A.dS0[(bh * dv + j0 + r) * DK + lane + 32 * i] = ds[r][i];
    }
}

template <typename Tin, int MODE, int DK>
cudaError_t launch_bwd_typed(const BwdArgs& a, int BH, size_t ntok, int mode, cudaStream_t stream) {
    const dim3 grid(a.dv_ / kBwdRowsPerCta, BH);
    cudaError_t err;
    if (grid.x > 1) {  // the CTAs of a head add their row sums into zeroed outputs
        if ((err = cudaMemsetAsync(a.dq, 0, ntok * DK * sizeof(float), stream)) != cudaSuccess) return err;
        if ((err = cudaMemsetAsync(a.dk, 0, ntok * DK * sizeof(float), stream)) != cudaSuccess) return err;
        if ((err = cudaMemsetAsync(a.dbeta, 0, ntok * sizeof(float), stream)) != cudaSuccess) return err;
        if (mode != GDR_DECAY_NONE &&
            (err = cudaMemsetAsync(a.dg, 0, ntok * (mode == GDR_DECAY_CHANNEL ? DK : 1) * sizeof(float), stream)) !=
                cudaSuccess)
            return err;
    }
    bwd_history_kernel<Tin, MODE, DK><<<dim3(a.dv_ / kHistRowsPerCta, BH), kBwdThreads, 0, stream>>>(a);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    profile_after_launch(stream);
    auto kern = bwd_reverse_kernel<Tin, MODE, DK>;
    const size_t smem = ((size_t)2 * kBwdWarps * (3 * DK + 2) + (size_t)kBwdStages * kBwdRowsPerCta * DK) * sizeof(float);
    if ((err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
        return err;
    kern<<<grid, kBwdThreads, smem, stream>>>(a);
    profile_after_launch(stream);
    return cudaGetLastError();
}

template <typename Tin, int MODE>
cudaError_t launch_bwd_dk(const BwdArgs& a, int dk, int BH, size_t ntok, cudaStream_t stream) {
    switch (dk) {
        case 32: return launch_bwd_typed<Tin, MODE, 32>(a, BH, ntok, MODE, stream);
        case 64: return launch_bwd_typed<Tin, MODE, 64>(a, BH, ntok, MODE, stream);
        case 128: return launch_bwd_typed<Tin, MODE, 128>(a, BH, ntok, MODE, stream);
        default: return cudaErrorInvalidValue;
    }
}

template <typename Tin>
cudaError_t launch_bwd_mode(const BwdArgs& a, int mode, int dk, int BH, size_t ntok, cudaStream_t stream) {
    switch (mode) {
        case GDR_DECAY_NONE: return launch_bwd_dk<Tin, GDR_DECAY_NONE>(a, dk, BH, ntok, stream);
        case GDR_DECAY_SCALAR: return launch_bwd_dk<Tin, GDR_DECAY_SCALAR>(a, dk, BH, ntok, stream);
        case GDR_DECAY_CHANNEL: return launch_bwd_dk<Tin, GDR_DECAY_CHANNEL>(a, dk, BH, ntok, stream);
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
              p.dg, p.dbeta, p.dS0, static_cast<float*>(p.workspace), p.T, p.H, p.dv_dim, p.scale, p.status};
    const int BH = p.B * p.H;
    const size_t ntok = (size_t)BH * p.T;
    if (p.dtype == GDR_BF16) return launch_bwd_mode<__nv_bfloat16>(a, p.mode, p.dk_dim, BH, ntok, stream);
    return launch_bwd_mode<float>(a, p.mode, p.dk_dim, BH, ntok, stream);
}

}  // namespace gdr
