// gdr_decode.cu -- one recurrent step of the gated delta rule for a batch of fp32 states.
//
// The decoding view ("linear attention and its gated descendants", Recurrent Linear Attention
// for Inference): each new token updates a constant-size state and reads it once. Per head,
// row j of S (s_j in R^{d_k}) needs only k, q, alpha, beta and v_j:
//
//   s_bar = s_j * alpha;  p = s_bar . k;  a = s_bar . q;  delta = beta (v_j - p)
//   o_j   = scale (a + delta (k . q));    s_j <- s_bar + delta k
//
// (a + delta (k.q) is the read of the updated row, (s_bar + delta k) . q, taken in the same pass).
// The step is bound by HBM: S is read once and written once (2 * 4 * d_k * d_v bytes per head).
// Layout of the work: 16 lanes own one row for d_k >= 128, 8 below (d_k / 16 or d_k / 8 consecutive
// floats each, 16-byte vector loads, so a warp touches whole rows per instruction, fully coalesced);
// the two dot products are reduced across those lanes with xor-shuffles. One CTA of 256 threads
// per (b, h); each thread carries two rows in flight. S is streamed with evict-first hints. At
// d_k = 128, 16 lanes a row hold 8 floats each: 64 registers a thread, four CTAs per SM (8 lanes:
// 102 registers, two CTAs) -- 105.2 -> 86.2 us per step at B = 256, H = 16.
//
// Gated DeltaNet-2 (EW; "Linear Attention Architectures: Mechanisms, Trade-offs, and Cross-Layer
// Routing", Sec. 3): an erase gate e [d_k] and a write gate w [d_v] replace beta:
//   p = s_bar . (e (.) k);  delta = w_j v_j - p;  s_j <- s_bar + delta k;  o_j = scale (a + delta (k . q)).
#include "gdr_internal.cuh"

namespace gdr {
namespace {

constexpr int kThreads = 256;
// lanes per state row: 16 for d_k >= 128 (8 floats a lane: fewer registers, more CTAs per SM), else 8
template <int DK>
constexpr int lanes_per_row() { return DK >= 128 ? 16 : 8; }

template <typename Tin, int N>
__device__ __forceinline__ void load_vec(const Tin* p, float (&x)[N]) {
#pragma unroll
    for (int i = 0; i < N; ++i) x[i] = load_f32(p + i);
}

template <int N>
__device__ __forceinline__ void load_row(const float* p, float (&x)[N]) {
    static_assert(N % 4 == 0, "row slice must be whole float4s");
#pragma unroll
    for (int i = 0; i < N; i += 4) {
        const float4 t = __ldcs(reinterpret_cast<const float4*>(p + i));
        x[i] = t.x; x[i + 1] = t.y; x[i + 2] = t.z; x[i + 3] = t.w;
    }
}

template <int N>
__device__ __forceinline__ void store_row(float* p, const float (&x)[N]) {
#pragma unroll
    for (int i = 0; i < N; i += 4) __stcs(reinterpret_cast<float4*>(p + i), make_float4(x[i], x[i + 1], x[i + 2], x[i + 3]));
}

// sum over the LPR lanes of a row group
template <int LPR>
__device__ __forceinline__ float group_sum(float x) {
#pragma unroll
    for (int m = 1; m < LPR; m <<= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
    return x;
}

template <typename Tin, typename Tout, int MODE, int DK, bool EW>
__global__ void __launch_bounds__(kThreads)
decode_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
              const float* __restrict__ g, const float* __restrict__ beta, float* __restrict__ S,
              Tout* __restrict__ o, int dv, float scale, int H, int pro, const float* __restrict__ gate_scale,
              const float* __restrict__ erase, const float* __restrict__ write) {
    constexpr int kLanesPerRow = lanes_per_row<DK>();
    constexpr int kRowsPerPass = kThreads / kLanesPerRow;
    constexpr int EPL = DK / kLanesPerRow;  // floats of a row per lane
    const size_t bh = blockIdx.x;
    const int sub = threadIdx.x & (kLanesPerRow - 1);
    const int row0 = threadIdx.x / kLanesPerRow;
    const int c0 = sub * EPL;
    float* Sh = S + bh * (size_t)dv * DK;
    // Loop bounds are uniform across a warp (its 4 rows share `jb`), so every lane reaches the
    // full-mask shuffles; rows past d_v are masked.
    const int warp_row0 = (threadIdx.x >> 5) * (32 / kLanesPerRow);
    const int lane_row = row0 - warp_row0;
    // the two state rows of pass jb (rows jb + lane_row and that + kRowsPerPass), zero past d_v
    auto load_pass = [&](int jb, float (&a)[EPL], float (&b)[EPL]) {
        const int j = jb + lane_row, j2 = j + kRowsPerPass;
#pragma unroll
        for (int i = 0; i < EPL; ++i) { a[i] = 0.f; b[i] = 0.f; }
        if (j < dv) load_row(Sh + (size_t)j * DK + c0, a);
        if (j2 < dv) load_row(Sh + (size_t)j2 * DK + c0, b);
    };
    // the state is nearly all of the traffic: the first pass's rows are requested before the token's
    // inputs, so that their latency overlaps the prologue
    float s1[EPL], s2[EPL];
    load_pass(warp_row0, s1, s2);

    float kr[EPL], qr[EPL], al[EPL];
    load_vec(k + bh * DK + c0, kr);
    load_vec(q + bh * DK + c0, qr);
    if (pro & GDR_PRO_L2NORM_QK) {  // the 8 lanes of a row group hold all of k and q
        float sk = 0.f, sq = 0.f;
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
            sk = fmaf(kr[i], kr[i], sk);
            sq = fmaf(qr[i], qr[i], sq);
        }
        const float nk = pro_inv_norm(group_sum<kLanesPerRow>(sk)), nq = pro_inv_norm(group_sum<kLanesPerRow>(sq));
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
            kr[i] *= nk;
            qr[i] *= nq;
        }
    }
    const bool gate = (pro & GDR_PRO_GATE_SOFTPLUS) != 0;
    const float A = (gate && gate_scale != nullptr) ? gate_scale[bh % (size_t)H] : 1.f;
    if (MODE == GDR_DECAY_CHANNEL) {
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
            const float x = g[bh * DK + c0 + i];
            al[i] = expf(gate ? pro_gate(x, A) : x);
        }
    } else {
        float a = 1.f;
        if (MODE == GDR_DECAY_SCALAR) a = expf(gate ? pro_gate(g[bh], A) : g[bh]);
#pragma unroll
        for (int i = 0; i < EPL; ++i) al[i] = a;
    }
    float kq = 0.f;
#pragma unroll
    for (int i = 0; i < EPL; ++i) kq = fmaf(kr[i], qr[i], kq);
    kq = group_sum<kLanesPerRow>(kq);
    float bt = 1.f;
    float er[EPL];  // the erase direction e (.) k (Gated DeltaNet-2)
    if (EW) {
#pragma unroll
        for (int i = 0; i < EPL; ++i) er[i] = erase[bh * DK + c0 + i] * kr[i];
    } else {
        bt = (pro & GDR_PRO_BETA_SIGMOID) ? pro_sigmoid(beta[bh]) : beta[bh];
    }
    for (int jb = warp_row0; jb < dv; jb += 2 * kRowsPerPass) {
        const int j = jb + lane_row;
        const int j2 = j + kRowsPerPass;
        const bool ok1 = j < dv;
        const bool ok2 = j2 < dv;
        if (jb != warp_row0) load_pass(jb, s1, s2);
        float v1 = ok1 ? load_f32(v + bh * dv + j) : 0.f;
        float v2 = ok2 ? load_f32(v + bh * dv + j2) : 0.f;
        if (EW) {  // the gated write target
            if (ok1) v1 *= write[bh * dv + j];
            if (ok2) v2 *= write[bh * dv + j2];
        }
        float p1 = 0.f, a1 = 0.f, p2 = 0.f, a2 = 0.f;
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
            const float rd = EW ? er[i] : kr[i];  // read direction of the prediction
            s1[i] *= al[i];
            p1 = fmaf(s1[i], rd, p1);
            a1 = fmaf(s1[i], qr[i], a1);
            s2[i] *= al[i];
            p2 = fmaf(s2[i], rd, p2);
            a2 = fmaf(s2[i], qr[i], a2);
        }
        p1 = group_sum<kLanesPerRow>(p1);
        a1 = group_sum<kLanesPerRow>(a1);
        p2 = group_sum<kLanesPerRow>(p2);
        a2 = group_sum<kLanesPerRow>(a2);
        const float d1 = bt * (v1 - p1);
        const float d2 = bt * (v2 - p2);
        if (sub == 0) {
            if (ok1) store_f32(o + bh * dv + j, scale * fmaf(d1, kq, a1));
            if (ok2) store_f32(o + bh * dv + j2, scale * fmaf(d2, kq, a2));
        }
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
            s1[i] = fmaf(d1, kr[i], s1[i]);
            s2[i] = fmaf(d2, kr[i], s2[i]);
        }
        if (ok1) store_row(Sh + (size_t)j * DK + c0, s1);
        if (ok2) store_row(Sh + (size_t)j2 * DK + c0, s2);
    }
}

template <typename Tin, typename Tout, int MODE, bool EW>
cudaError_t launch_mode_ew(const DecodeProblem& p, cudaStream_t stream) {
    const dim3 grid((unsigned)((size_t)p.B * p.H));
    const Tin* q = static_cast<const Tin*>(p.q);
    const Tin* k = static_cast<const Tin*>(p.k);
    const Tin* v = static_cast<const Tin*>(p.v);
    Tout* o = static_cast<Tout*>(p.o);
    switch (p.dk) {
        case 32: decode_kernel<Tin, Tout, MODE, 32, EW><<<grid, kThreads, 0, stream>>>(q, k, v, p.g, p.beta, p.S, o, p.dv, p.scale, p.H, p.prologue, p.gate_scale, p.erase, p.write); break;
        case 64: decode_kernel<Tin, Tout, MODE, 64, EW><<<grid, kThreads, 0, stream>>>(q, k, v, p.g, p.beta, p.S, o, p.dv, p.scale, p.H, p.prologue, p.gate_scale, p.erase, p.write); break;
        case 128: decode_kernel<Tin, Tout, MODE, 128, EW><<<grid, kThreads, 0, stream>>>(q, k, v, p.g, p.beta, p.S, o, p.dv, p.scale, p.H, p.prologue, p.gate_scale, p.erase, p.write); break;
        case 256: decode_kernel<Tin, Tout, MODE, 256, EW><<<grid, kThreads, 0, stream>>>(q, k, v, p.g, p.beta, p.S, o, p.dv, p.scale, p.H, p.prologue, p.gate_scale, p.erase, p.write); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

template <typename Tin, typename Tout, int MODE>
cudaError_t launch_mode(const DecodeProblem& p, cudaStream_t stream) {
    return p.erase != nullptr ? launch_mode_ew<Tin, Tout, MODE, true>(p, stream)
                              : launch_mode_ew<Tin, Tout, MODE, false>(p, stream);
}

template <typename Tin, typename Tout>
cudaError_t launch_dtype(const DecodeProblem& p, cudaStream_t stream) {
    switch (p.mode) {
        case GDR_DECAY_NONE: return launch_mode<Tin, Tout, GDR_DECAY_NONE>(p, stream);
        case GDR_DECAY_SCALAR: return launch_mode<Tin, Tout, GDR_DECAY_SCALAR>(p, stream);
        case GDR_DECAY_CHANNEL: return launch_mode<Tin, Tout, GDR_DECAY_CHANNEL>(p, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

bool decode_supported(int dk, int dv) {
    return (dk == 32 || dk == 64 || dk == 128 || dk == 256) && dv >= 1;
}

cudaError_t launch_decode(const DecodeProblem& p, cudaStream_t stream) {
    if (p.dtype == GDR_BF16 && p.o_dtype == GDR_BF16) return launch_dtype<__nv_bfloat16, __nv_bfloat16>(p, stream);
    if (p.dtype == GDR_BF16 && p.o_dtype == GDR_F32) return launch_dtype<__nv_bfloat16, float>(p, stream);
    if (p.dtype == GDR_F32 && p.o_dtype == GDR_F32) return launch_dtype<float, float>(p, stream);
    return cudaErrorInvalidValue;
}

}  // namespace gdr
