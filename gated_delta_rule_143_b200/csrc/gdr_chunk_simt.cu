// gdr_chunk_simt.cu -- chunked gated delta-rule forward on the CUDA cores in fp32.
//
// This is the exact-precision path (fp32 inputs, fp32 arithmetic, no TF32) and the path for
// shapes the tensor-core kernel does not take. One CTA owns a slice of DVS rows of one head's
// state S (rows of S evolve independently given k, beta and alpha) and walks the chunks of
// that head in order. Per chunk of n <= C tokens (Gamma = inclusive cumulative log-decay,
// gamma = exp(Gamma)):
//
//   A_ri  = beta_r sum_c k_rc k_ic exp(Gamma_rc - Gamma_ic)   (i < r)   strictly lower
//   P_ri  =        sum_c q_rc k_ic exp(Gamma_rc - Gamma_ic)   (i <= r)  causal incl. diagonal
//   R     = diag(beta) (V - (K*gamma) S^T)                    right-hand side
//   Delta = (I + A)^-1 R                                      forward substitution
//   O     = scale [ (Q*gamma) S^T + P Delta ]
//   S    <- S Diag(gamma_n) + Delta^T (K * gamma_n / gamma)
//
// which is the chunk form of "linear attention and its gated descendants" (Chunkwise
// Parallel Form) with the WY/UT compact form of a chunk of delta-rule updates ("Linear
// Attention & DeltaNet", item 3): (I + A)^-1 applied to R gives U - W S^T directly.
// Pairwise decays exp(Gamma_r - Gamma_i) with i <= r never exceed 1, so any g <= 0 is safe.
//
// Gated DeltaNet-2 (EW = true; "Linear Attention Architectures: Mechanisms, Trade-offs, and
// Cross-Layer Routing", Sec. 3): a channel-wise erase gate e on the key side and write gate w on the
// value side replace beta, S_t = S_bar + (w (.) v - S_bar (e (.) k)) k^T with S_bar = S_{t-1} Diag(alpha).
// In the chunk form the erase direction E = e (.) K takes the place of diag(beta) K on the left of the
// Gram and of the state read, and the write target w (.) V that of diag(beta) V:
//   A_ri = sum_c E_rc k_ic exp(Gamma_rc - Gamma_ic) (i < r),  R = w (.) V - (E*gamma) S^T.
#include "gdr_internal.cuh"

namespace gdr {
namespace {

constexpr int kC = 64;        // chunk length
constexpr int kDVS = 32;      // state rows per CTA
constexpr int kThreads = 256;

template <int DK, bool EW = false>
struct SimtSmem {
    static constexpr int kLd = DK + 1;        // padded row stride of K, Q, Gamma, S
    static constexpr int kLdC = kC + 1;       // padded stride of A, P
    static constexpr int kLdV = kDVS + 1;     // padded stride of the value slice
    static constexpr size_t floats =
        2 * kC * kLd          // K, Q
        + kC * kLd            // Gamma (per channel; scalar mode uses column 0)
        + kDVS * kLd          // S slice
        + 2 * kC * kLdV       // R/Delta, O_inter
        + 2 * kC * kLdC       // A, P
        + 2 * kC              // beta, tail decay (scalar)
        + (EW ? kC * kLd : 0);  // erase directions e (.) k (Gated DeltaNet-2)
    static constexpr size_t bytes = floats * sizeof(float);
};

template <typename Tin, typename Tout, int MODE, int DK, bool EW>
__global__ void __launch_bounds__(kThreads)
chunk_simt_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
                  const float* __restrict__ g, const float* __restrict__ beta, const float* S0,
                  Tout* __restrict__ o, float* S_T, int T, int H, int dv, float scale, int pro,
                  const float* __restrict__ gate_scale, const float* __restrict__ erase,
                  const float* __restrict__ write) {
    using L = SimtSmem<DK, EW>;
    extern __shared__ float smem[];
    float* sK = smem;
    float* sQ = sK + kC * L::kLd;
    float* sG = sQ + kC * L::kLd;
    float* sS = sG + kC * L::kLd;
    float* sR = sS + kDVS * L::kLd;
    float* sOi = sR + kC * L::kLdV;
    float* sA = sOi + kC * L::kLdV;
    float* sP = sA + kC * L::kLdC;
    float* sBeta = sP + kC * L::kLdC;
    float* sTail = sBeta + kC;
    float* sE = sTail + kC;  // EW only: e (.) k, [kC][kLd]

    const int tid = threadIdx.x;
    const int j0 = blockIdx.x * kDVS;           // first state row of this CTA
    const int h = blockIdx.y;
    const int b = blockIdx.z;
    const int nrows = min(kDVS, dv - j0);
    const size_t bh = (size_t)b * H + h;
    const bool gate = (pro & GDR_PRO_GATE_SOFTPLUS) != 0;
    const float A = (gate && gate_scale != nullptr) ? gate_scale[h] : 1.f;

    // initial state slice
    for (int idx = tid; idx < kDVS * DK; idx += kThreads) {
        const int j = idx / DK, c = idx % DK;
        float s = 0.f;
        if (S0 != nullptr && j < nrows) s = S0[(bh * dv + j0 + j) * DK + c];
        sS[j * L::kLd + c] = s;
    }

    for (int c0 = 0; c0 < T; c0 += kC) {
        const int n = min(kC, T - c0);
        __syncthreads();
        // ---- stage the chunk: K, Q, value slice, beta, cumulative log-decay
        for (int idx = tid; idx < n * DK; idx += kThreads) {
            const int r = idx / DK, c = idx % DK;
            const size_t tok = ((size_t)b * T + c0 + r) * H + h;
            const float kv = load_f32(k + tok * DK + c);
            sK[r * L::kLd + c] = kv;
            sQ[r * L::kLd + c] = load_f32(q + tok * DK + c);
            if (EW) sE[r * L::kLd + c] = erase[tok * DK + c] * kv;
        }
        for (int idx = tid; idx < n * kDVS; idx += kThreads) {
            const int r = idx / kDVS, j = idx % kDVS;
            const size_t tok = ((size_t)b * T + c0 + r) * H + h;
            float x = 0.f;
            if (j < nrows) {
                x = load_f32(v + tok * dv + j0 + j);
                if (EW) x *= write[tok * dv + j0 + j];  // the gated write target
            }
            sR[r * L::kLdV + j] = x;
        }
        for (int r = tid; r < n; r += kThreads) {
            const float x = EW ? 1.f : beta[((size_t)b * T + c0 + r) * H + h];
            sBeta[r] = (pro & GDR_PRO_BETA_SIGMOID) ? pro_sigmoid(x) : x;
        }
        if (MODE == GDR_DECAY_SCALAR) {
            if (tid == 0) {
                float acc = 0.f;
                for (int r = 0; r < n; ++r) {
                    const float x = g[((size_t)b * T + c0 + r) * H + h];
                    acc += gate ? pro_gate(x, A) : x;
                    sG[r * L::kLd] = acc;
                }
            }
        } else if (MODE == GDR_DECAY_CHANNEL) {
            for (int c = tid; c < DK; c += kThreads) {
                float acc = 0.f;
                for (int r = 0; r < n; ++r) {
                    const float x = g[(((size_t)b * T + c0 + r) * H + h) * DK + c];
                    acc += gate ? pro_gate(x, A) : x;
                    sG[r * L::kLd + c] = acc;
                }
            }
        }
        __syncthreads();
        if (pro & GDR_PRO_L2NORM_QK) {  // one warp per row of K and of Q
            const int lane = tid & 31;
            for (int rr = tid >> 5; rr < 2 * n; rr += kThreads / 32) {
                float* row = (rr < n ? sK : sQ) + (rr % n) * L::kLd;
                float ss = 0.f;
                for (int c = lane; c < DK; c += 32) ss = fmaf(row[c], row[c], ss);
#pragma unroll
                for (int m = 16; m > 0; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
                const float inv = pro_inv_norm(ss);
                for (int c = lane; c < DK; c += 32) row[c] *= inv;
            }
            __syncthreads();
        }
        if (MODE == GDR_DECAY_SCALAR) {
            for (int i = tid; i < n; i += kThreads) sTail[i] = expf(sG[(n - 1) * L::kLd] - sG[i * L::kLd]);
        }

        // ---- A (strictly lower, beta_r folded in) and P (causal incl. diagonal)
        for (int idx = tid; idx < kC * kC; idx += kThreads) {
            const int r = idx / kC, i = idx % kC;
            float a = 0.f, p = 0.f;
            if (r < n && i <= r) {
                const float* kr = (EW ? sE : sK) + r * L::kLd;  // erase direction of row r
                const float* ki = sK + i * L::kLd;
                const float* qr = sQ + r * L::kLd;
                if (MODE == GDR_DECAY_CHANNEL) {
                    const float* Gr = sG + r * L::kLd;
                    const float* Gi = sG + i * L::kLd;
                    for (int c = 0; c < DK; ++c) {
                        const float kid = ki[c] * expf(Gr[c] - Gi[c]);
                        a = fmaf(kr[c], kid, a);
                        p = fmaf(qr[c], kid, p);
                    }
                } else {
                    for (int c = 0; c < DK; ++c) {
                        a = fmaf(kr[c], ki[c], a);
                        p = fmaf(qr[c], ki[c], p);
                    }
                    if (MODE == GDR_DECAY_SCALAR) {
                        const float d = expf(sG[r * L::kLd] - sG[i * L::kLd]);
                        a *= d;
                        p *= d;
                    }
                }
                a = (i < r) ? sBeta[r] * a : 0.f;
            }
            sA[r * L::kLdC + i] = a;
            sP[r * L::kLdC + i] = p;
        }

        // ---- R = diag(beta)(V - (K*gamma) S^T) and O_inter = (Q*gamma) S^T
        for (int idx = tid; idx < n * kDVS; idx += kThreads) {
            const int r = idx / kDVS, j = idx % kDVS;
            const float* kr = (EW ? sE : sK) + r * L::kLd;  // the state is read along the erase direction
            const float* qr = sQ + r * L::kLd;
            const float* sj = sS + j * L::kLd;
            float x = 0.f, y = 0.f;
            if (MODE == GDR_DECAY_CHANNEL) {
                const float* Gr = sG + r * L::kLd;
                for (int c = 0; c < DK; ++c) {
                    const float sg = sj[c] * expf(Gr[c]);
                    x = fmaf(kr[c], sg, x);
                    y = fmaf(qr[c], sg, y);
                }
            } else {
                for (int c = 0; c < DK; ++c) {
                    x = fmaf(kr[c], sj[c], x);
                    y = fmaf(qr[c], sj[c], y);
                }
                if (MODE == GDR_DECAY_SCALAR) {
                    const float gr = expf(sG[r * L::kLd]);
                    x *= gr;
                    y *= gr;
                }
            }
            sR[r * L::kLdV + j] = sBeta[r] * (sR[r * L::kLdV + j] - x);
            sOi[r * L::kLdV + j] = y;
        }
        __syncthreads();

        // ---- forward substitution Delta = (I + A)^-1 R; 8 lanes cooperate on one column
        {
            const int j = tid >> 3;        // column 0..31
            const int sub = tid & 7;
            for (int r = 1; r < n; ++r) {
                float part = 0.f;
                for (int i = sub; i < r; i += 8) part = fmaf(sA[r * L::kLdC + i], sR[i * L::kLdV + j], part);
                part += __shfl_xor_sync(0xffffffffu, part, 1);
                part += __shfl_xor_sync(0xffffffffu, part, 2);
                part += __shfl_xor_sync(0xffffffffu, part, 4);
                if (sub == 0) sR[r * L::kLdV + j] -= part;
                __syncwarp();
            }
        }
        __syncthreads();

        // ---- output O = scale [O_inter + P Delta]
        for (int idx = tid; idx < n * kDVS; idx += kThreads) {
            const int r = idx / kDVS, j = idx % kDVS;
            if (j >= nrows) continue;
            float acc = sOi[r * L::kLdV + j];
            for (int i = 0; i <= r; ++i) acc = fmaf(sP[r * L::kLdC + i], sR[i * L::kLdV + j], acc);
            const size_t tok = ((size_t)b * T + c0 + r) * H + h;
            store_f32(o + tok * dv + j0 + j, scale * acc);
        }

        // ---- state S <- S Diag(gamma_n) + Delta^T (K * gamma_n / gamma)
        for (int idx = tid; idx < kDVS * DK; idx += kThreads) {
            const int j = idx / DK, c = idx % DK;
            float s = sS[j * L::kLd + c];
            if (MODE == GDR_DECAY_CHANNEL) {
                const float Gn = sG[(n - 1) * L::kLd + c];
                s *= expf(Gn);
                for (int i = 0; i < n; ++i)
                    s = fmaf(sR[i * L::kLdV + j], sK[i * L::kLd + c] * expf(Gn - sG[i * L::kLd + c]), s);
            } else if (MODE == GDR_DECAY_SCALAR) {
                s *= expf(sG[(n - 1) * L::kLd]);
                for (int i = 0; i < n; ++i) s = fmaf(sR[i * L::kLdV + j] * sTail[i], sK[i * L::kLd + c], s);
            } else {
                for (int i = 0; i < n; ++i) s = fmaf(sR[i * L::kLdV + j], sK[i * L::kLd + c], s);
            }
            sS[j * L::kLd + c] = s;
        }
    }
    __syncthreads();
    if (S_T != nullptr) {
        for (int idx = tid; idx < nrows * DK; idx += kThreads) {
            const int j = idx / DK, c = idx % DK;
            S_T[(bh * dv + j0 + j) * DK + c] = sS[j * L::kLd + c];
        }
    }
}

// ------------------------------------------------------------- short sequences --
// Up to kRecMaxT tokens the token-by-token recurrence itself beats the chunk form's per-chunk
// work: one warp per state row (rows of S evolve independently given k, beta and alpha), the row
// in registers (lane holds columns lane + 32 i). Per token, with alpha = exp(g):
//   s <- s * alpha;  p = s . k;  s <- s + beta (v_j - p) k;  o_j = scale (s . q)
// (the delta rule of "Linear Attention & DeltaNet" with the gate of "linear attention and its
// gated descendants"). Tokens are staged in shared memory kRecTB at a time; the next block's
// loads are in flight while the current one is computed.
constexpr int kRecWarps = 8;   // state rows per CTA
constexpr int kRecTB = 16;     // tokens per staged block
constexpr int kRecMaxT = 256;  // sequences up to this length run the recurrence

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
    return x;
}

template <typename Tin, typename Tout, int MODE, int DK, bool EW>
__global__ void __launch_bounds__(kRecWarps * 32)
recurrent_simt_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
                      const float* __restrict__ g, const float* __restrict__ beta, const float* S0,
                      Tout* __restrict__ o, float* S_T, int T, int H, int dv, float scale, int pro,
                      const float* __restrict__ gate_scale, const float* __restrict__ erase,
                      const float* __restrict__ write) {
    constexpr int NT = kRecWarps * 32;
    constexpr int NL = DK / 32;                                  // state columns per lane
    constexpr int NA = MODE == GDR_DECAY_CHANNEL ? DK : 1;       // decay factors per token
    constexpr int KPT = kRecTB * DK / NT;                        // staged k (and q) values per thread
    static_assert(kRecTB * DK % NT == 0 && kRecTB * kRecWarps <= NT && kRecTB <= NT, "staging split");
    constexpr int NE = EW ? DK : 1;  // Gated DeltaNet-2: erase directions e (.) k
    __shared__ float sK[kRecTB][DK], sQ[kRecTB][DK], sAl[kRecTB][NA], sV[kRecTB][kRecWarps], sB[kRecTB];
    __shared__ float sE[kRecTB][NE];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int j0 = blockIdx.x * kRecWarps, j = j0 + warp;       // this warp's state row
    const int h = blockIdx.y, b = blockIdx.z;
    const size_t bh = (size_t)b * H + h;
    const bool active = j < dv;
    auto tok_of = [&](int t) { return ((size_t)b * T + t) * H + h; };
    const bool gate = (pro & GDR_PRO_GATE_SOFTPLUS) != 0;
    const float A = (gate && gate_scale != nullptr) ? gate_scale[h] : 1.f;

    // one block's inputs, held in registers between its load and its store into shared memory:
    // thread tid holds k, q (and the channel gate's g) at flat index tid + NT m of the block, the
    // value of (token tid / kRecWarps, row j0 + tid % kRecWarps), and beta (and the scalar g) of
    // token tid
    float rk[KPT], rq[KPT], rg[KPT], re[KPT], rv = 0.f, rb = 0.f, rs = 0.f;
    auto load_block = [&](int t0) {
        const int n = min(kRecTB, T - t0);
#pragma unroll
        for (int m = 0; m < KPT; ++m) {
            const int idx = tid + NT * m, r = idx / DK, c = idx % DK;
            rk[m] = rq[m] = rg[m] = re[m] = 0.f;
            if (r < n) {
                const size_t tok = tok_of(t0 + r);
                rk[m] = load_f32(k + tok * DK + c);
                rq[m] = load_f32(q + tok * DK + c);
                if (MODE == GDR_DECAY_CHANNEL) rg[m] = g[tok * DK + c];
                if (EW) re[m] = erase[tok * DK + c];
            }
        }
        const int rr = tid / kRecWarps, w = tid % kRecWarps;
        rv = (rr < n && j0 + w < dv) ? load_f32(v + tok_of(t0 + rr) * dv + j0 + w) : 0.f;
        if (EW && rr < n && j0 + w < dv) rv *= write[tok_of(t0 + rr) * dv + j0 + w];  // gated write target
        if (tid < n) {
            rb = EW ? 1.f : beta[tok_of(t0 + tid)];
            if (MODE == GDR_DECAY_SCALAR) rs = g[tok_of(t0 + tid)];
        }
    };
    auto store_block = [&]() {
#pragma unroll
        for (int m = 0; m < KPT; ++m) {
            const int idx = tid + NT * m, r = idx / DK, c = idx % DK;
            sK[r][c] = rk[m];
            sQ[r][c] = rq[m];
            if (EW) sE[r][c] = re[m] * rk[m];
            if (MODE == GDR_DECAY_CHANNEL) sAl[r][c] = expf(gate ? pro_gate(rg[m], A) : rg[m]);
        }
        if (tid < kRecTB * kRecWarps) sV[tid / kRecWarps][tid % kRecWarps] = rv;
        if (tid < kRecTB) {
            sB[tid] = (pro & GDR_PRO_BETA_SIGMOID) ? pro_sigmoid(rb) : rb;
            if (MODE == GDR_DECAY_SCALAR) sAl[tid][0] = expf(gate ? pro_gate(rs, A) : rs);
        }
    };
    // L2 normalisation of the staged k and q vectors (rows past the sequence are zero and stay so):
    // warp w takes tokens w and w + kRecWarps; each warp rescales only its own rows
    auto normalise_block = [&]() {
#pragma unroll
        for (int r = warp; r < kRecTB; r += kRecWarps) {
            float sk = 0.f, sq = 0.f;
#pragma unroll
            for (int i = 0; i < NL; ++i) {
                sk = fmaf(sK[r][lane + 32 * i], sK[r][lane + 32 * i], sk);
                sq = fmaf(sQ[r][lane + 32 * i], sQ[r][lane + 32 * i], sq);
            }
            const float nk = pro_inv_norm(warp_sum(sk)), nq = pro_inv_norm(warp_sum(sq));
#pragma unroll
            for (int i = 0; i < NL; ++i) {
                sK[r][lane + 32 * i] *= nk;
                sQ[r][lane + 32 * i] *= nq;
            }
        }
    };
    const bool norm = (pro & GDR_PRO_L2NORM_QK) != 0;

    float s[NL];
#pragma unroll
    for (int i = 0; i < NL; ++i) s[i] = (active && S0 != nullptr) ? S0[(bh * dv + j) * DK + lane + 32 * i] : 0.f;
    load_block(0);
    store_block();
    __syncthreads();
    if (norm) {
        normalise_block();
        __syncthreads();
    }
    for (int t0 = 0; t0 < T; t0 += kRecTB) {
        const int n = min(kRecTB, T - t0);
        if (t0 + kRecTB < T) load_block(t0 + kRecTB);  // in flight while this block is computed
        if (active) {
            // the state's chain carries one reduction per token (s . k); the lane partials of the
            // outputs s . q are reduced after the block, 16 independent reductions at once
            float ap[kRecTB];
#pragma unroll
            for (int r = 0; r < kRecTB; ++r) {
                ap[r] = 0.f;
                if (r < n) {
                    float kk[NL], p = 0.f;
#pragma unroll
                    for (int i = 0; i < NL; ++i) {
                        kk[i] = sK[r][lane + 32 * i];
                        if (MODE == GDR_DECAY_SCALAR) s[i] *= sAl[r][0];
                        if (MODE == GDR_DECAY_CHANNEL) s[i] *= sAl[r][lane + 32 * i];
                        p = fmaf(s[i], EW ? sE[r][(lane + 32 * i) % NE] : kk[i], p);  // read along e (.) k
                    }
                    p = warp_sum(p);
                    const float d = sB[r] * (sV[r][warp] - p);
#pragma unroll
                    for (int i = 0; i < NL; ++i) {
                        s[i] = fmaf(d, kk[i], s[i]);
                        ap[r] = fmaf(s[i], sQ[r][lane + 32 * i], ap[r]);
                    }
                }
            }
#pragma unroll
            for (int r = 0; r < kRecTB; ++r) ap[r] = warp_sum(ap[r]);
            float mine = 0.f;  // lane r writes the output of token r
#pragma unroll
            for (int r = 0; r < kRecTB; ++r)
                if (lane == r) mine = ap[r];
            if (lane < n) store_f32(o + tok_of(t0 + lane) * dv + j, scale * mine);
        }
        if (t0 + kRecTB < T) {
            __syncthreads();  // every warp is done with this block
            store_block();
            __syncthreads();
            if (norm) {
                normalise_block();
                __syncthreads();
            }
        }
    }
    if (active && S_T != nullptr) {
#pragma unroll
        for (int i = 0; i < NL; ++i) S_T[(bh * dv + j) * DK + lane + 32 * i] = s[i];
    }
}

template <typename Tin, typename Tout, int MODE, int DK, bool EW>
cudaError_t launch_typed_ew(const ChunkProblem& p, cudaStream_t stream) {
    if (p.T <= kRecMaxT) {
        dim3 grid((p.dv + kRecWarps - 1) / kRecWarps, p.H, p.B);
        recurrent_simt_kernel<Tin, Tout, MODE, DK, EW><<<grid, kRecWarps * 32, 0, stream>>>(
            static_cast<const Tin*>(p.q), static_cast<const Tin*>(p.k), static_cast<const Tin*>(p.v), p.g, p.beta,
            p.S0, static_cast<Tout*>(p.o), p.S_T, p.T, p.H, p.dv, p.scale, p.prologue, p.gate_scale, p.erase,
            p.write);
        profile_after_launch(stream);
        return cudaGetLastError();
    }
    auto kern = chunk_simt_kernel<Tin, Tout, MODE, DK, EW>;
    const size_t smem = SimtSmem<DK, EW>::bytes;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    dim3 grid((p.dv + kDVS - 1) / kDVS, p.H, p.B);
    kern<<<grid, kThreads, smem, stream>>>(
        static_cast<const Tin*>(p.q), static_cast<const Tin*>(p.k), static_cast<const Tin*>(p.v), p.g, p.beta,
        p.S0, static_cast<Tout*>(p.o), p.S_T, p.T, p.H, p.dv, p.scale, p.prologue, p.gate_scale, p.erase, p.write);
    profile_after_launch(stream);
    return cudaGetLastError();
}

template <typename Tin, typename Tout, int MODE, int DK>
cudaError_t launch_typed(const ChunkProblem& p, cudaStream_t stream) {
    return p.erase != nullptr ? launch_typed_ew<Tin, Tout, MODE, DK, true>(p, stream)
                              : launch_typed_ew<Tin, Tout, MODE, DK, false>(p, stream);
}

template <typename Tin, typename Tout, int MODE>
cudaError_t launch_mode(const ChunkProblem& p, cudaStream_t stream) {
    switch (p.dk) {
        case 32: return launch_typed<Tin, Tout, MODE, 32>(p, stream);
        case 64: return launch_typed<Tin, Tout, MODE, 64>(p, stream);
        case 128: return launch_typed<Tin, Tout, MODE, 128>(p, stream);
        default: return cudaErrorInvalidValue;
    }
}

template <typename Tin, typename Tout>
cudaError_t launch_dtype(const ChunkProblem& p, cudaStream_t stream) {
    switch (p.mode) {
        case GDR_DECAY_NONE: return launch_mode<Tin, Tout, GDR_DECAY_NONE>(p, stream);
        case GDR_DECAY_SCALAR: return launch_mode<Tin, Tout, GDR_DECAY_SCALAR>(p, stream);
        case GDR_DECAY_CHANNEL: return launch_mode<Tin, Tout, GDR_DECAY_CHANNEL>(p, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

bool chunk_simt_supported(int dk, int dv, int chunk) {
    return (dk == 32 || dk == 64 || dk == 128) && (dv == 32 || dv == 64 || dv == 128) && chunk == kC;
}

cudaError_t launch_chunk_simt(const ChunkProblem& p, cudaStream_t stream) {
    if (p.dtype == GDR_BF16 && p.o_dtype == GDR_BF16) return launch_dtype<__nv_bfloat16, __nv_bfloat16>(p, stream);
    if (p.dtype == GDR_BF16 && p.o_dtype == GDR_F32) return launch_dtype<__nv_bfloat16, float>(p, stream);
    if (p.dtype == GDR_F32 && p.o_dtype == GDR_F32) return launch_dtype<float, float>(p, stream);
    return cudaErrorInvalidValue;
}

}  // namespace gdr
