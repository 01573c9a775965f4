// gdr_chunk_tc.cu -- chunked gated delta-rule forward on the 5th-generation tensor cores.
//
// bf16 q/k/v, d_k = d_v = 128, chunk C = 64; fp16 MMA operands, fp32 accumulation and an fp32
// state, both in TMEM. The chunk form ("linear attention and its gated descendants", Chunkwise
// Parallel Form, with the WY/UT compact form of a chunk of delta-rule updates from "Linear
// Attention & DeltaNet", item 3), with Gamma the inclusive cumulative log-decay inside the chunk
// and gamma = exp(Gamma):
//
//   A  = strictly_lower(diag(beta) (K*gamma)(K/gamma)^T),  T = (I + A)^-1      (UT transform)
//   W  = T diag(beta) (K*gamma),  U = T diag(beta) V                           (WY factors)
//   P  = causal_incl_diag((Q*gamma)(K/gamma)^T)
//   Delta = U - W S^T
//   O  = scale [ (Q*gamma) S^T + P Delta ]
//   S <- S Diag(gamma_C) + Delta^T (K * gamma_C / gamma)
//
// Work split. A prep pass (one 256-thread pipeline per chunk, all chunks independent) computes the
// S-independent factors and writes them as ready-to-use, 128-byte-swizzled fp16 operand images
// (the "hand-off block"); a state pass (one 576-thread CTA per (b, h)) walks the chunks in order,
// copies each block into shared memory with bulk copies and runs the S-dependent MMAs; the fp32
// state is the TMEM accumulator of the state product and enters the other MMAs as an fp16 copy.
//
// Prep, per chunk: TMA loads of the bf16 K, Q, V tiles straight into the swizzled K-major layout;
// Gram products [K; Q] K^T on tcgen05 (bf16 operands for the scalar gate and DeltaNet, exact with
// fp32 accumulation; fp16 decay-factored operands for the channel gate); A and P from TMEM with the
// pairwise decays; T = (I + A)^-1 by forward substitution on 16x16 diagonal blocks and two levels
// of block merges on warp MMAs (tf32); then W = [T diag(beta); 0] (K*gamma) (M = 128, N = d_k) and
// U^T = V^T (T diag(beta))^T (M = d_v) on tcgen05.
//
// Decay handling: the scalar gate's Gram products are scaled elementwise by exp(Gamma_r - Gamma_i)
// <= 1 (safe for any g <= 0), computed as exp(Gamma_r) * exp(-Gamma_i) while every |Gamma| of the
// chunk stays within 120 log2 units (both factors normal fp32) and directly beyond that. The channel
// gate's factors are folded into the Gram operands around a mid-chunk reference,
// (K e^{Gamma - Gamma_ref})(K e^{Gamma_ref - Gamma})^T, for every key channel whose cumulative
// log-decay varies by at most kStrongSpread log2 units inside the chunk (factors within 2^14, far
// inside fp16); the other ("strong") channels are left out of the tensor-core product and their
// terms k_r,d k_i,d 2^(Gamma_r,d - Gamma_i,d) (each factor <= 1) are added to the Gram on the CUDA
// cores, in fp32, from a second copy of the bf16 tiles. Any g <= 0 is computed exactly.
//
// Prologue (gdr_chunk_fwd_ex): beta = sigmoid(logit) and g = -A softplus(a) are applied where the prep
// loads beta and g. For the L2 normalisation of q and k the prep takes the inverse norms of the 128
// rows of the [K; Q] tile after its TMA load and folds them in as row factors: into the hand-off
// images and the operands it builds from the tiles, and into the epilogue of the Gram products,
// which run on the raw bf16 tiles (x_ri * n_r * n_i), so no normalised copy is ever stored.
//
// Operands are fp16, not bf16: with bf16 operands the rounding of the intermediate factors alone
// exceeded the 2e-2 * rms(o) parity bar; fp16 holds the bf16 inputs exactly at these ranges and
// runs at the same tensor-core rate.
#include <cuda_fp16.h>

#include "gdr_sm100.cuh"

namespace gdr {
namespace {

using namespace sm100;

constexpr int kC = 64;    // chunk length
constexpr int kD = 128;   // d_k = d_v
constexpr float kLog2e = 1.4426950408889634f;

// ------------------------------------------------------------------ hand-off block --
// Per-chunk block in the workspace (byte offsets). Images are laid out exactly as the state
// pass's MMAs read them. Part A (double-buffered in the state pass) is [0, kPartA); U^T follows.
constexpr uint32_t kOffWQ = 0;          // [W; Q*gamma]  fp16 K-major, 128 rows (r | 64 + r) x 128 (d_k)
constexpr uint32_t kOffP = 32768;       // P             fp16 K-major, 64 rows (r) x 64 (i)
constexpr uint32_t kOffKT = 40960;      // K*gamma_C/gamma fp16 MN-major, 64 rows (i) x 128 (d_k)
constexpr uint32_t kOffGam = 57344;     // gamma_C       fp32 [128]
constexpr uint32_t kPartA = 57856;      // bytes of part A (multiple of 16)
constexpr uint32_t kPartWQ = kOffP;     // part A splits into [W; Q*gamma] and the rest (P, K~, gamma_C)
constexpr uint32_t kOffUT = 58368;      // U^T           fp16 K-major, 128 rows (d_v) x 64 (r)
constexpr uint32_t kHandoffStride = 74752;  // multiple of 1024

// ------------------------------------------------------------------ prep pipeline --
constexpr int kPrepThreads = 256;
// shared memory of one prep pipeline (offsets from a 1024-aligned base)
constexpr uint32_t kPKQ = 0;          // [K; Q] bf16 (TMA) K-major 128 x 128; K rows become K*gamma (fp16)
constexpr uint32_t kPV = 32768;       // V bf16 (TMA) K-major 64 x 128, converted in place to fp16
constexpr uint32_t kPTBZ = 49152;     // [T diag(beta); Z] fp16 K-major 64-row blocks (2 x 8 KiB)
constexpr uint32_t kPA = kPTBZ + 16384;  // A^T fp32 [64][kLdA]
constexpr int kLdA = 68;
constexpr uint32_t kPT = kPA + 64 * kLdA * 4;   // T fp32 [64][kLdT]
constexpr int kLdT = 68;
constexpr uint32_t kPX = kPT + 64 * kLdT * 4;   // merge scratch fp32 [32][kLdX]
constexpr int kLdX = 36;
constexpr uint32_t kPBeta = kPX + 32 * kLdX * 4;     // beta [64]
constexpr uint32_t kPGam = kPBeta + 256;             // Gamma * log2(e): [64] or [64][128] (channel)
constexpr uint32_t kPInvE = kPGam + 256;             // scalar gate: 2^-Gamma [64], then a "factorable" flag
constexpr uint32_t kPKB = (kPGam + 32768 + 1023) & ~1023u;  // channel: K'' fp16 K-major 64 x 128
// DeltaNet and the scalar gate: two regions take turns as the [K; Q] tile (32 KiB) and as A^T and T
// (2 x 17 KiB), so that the next task's tile loads while this task finishes; the solve's scratch
// sits in the tile's Q rows, free once the Gram product is done
constexpr uint32_t kFRegion = 2 * 64 * kLdA * 4;
static_assert(kLdA == kLdT && kFRegion >= 32768 && kFRegion % 1024 == 0, "a region holds A^T and T, or the tile");
static_assert(32 * kLdX * 4 <= 8192, "the solve's scratch fits in one 8 KiB box of Q rows");
constexpr uint32_t kFV = 2 * kFRegion;                // V bf16 (TMA) K-major 64 x 128
constexpr uint32_t kFTBZ = kFV + 16384;               // [T diag(beta); Z]
constexpr uint32_t kFBeta = kFTBZ + 16384;            // beta [64]
constexpr uint32_t kFGam = kFBeta + 256;              // Gamma * log2(e) [64]
constexpr uint32_t kFInvE = kFGam + 256;              // 2^-Gamma [64], then a "factorable" flag
constexpr uint32_t kPrepBytesScalar = (kFInvE + 512 + 512 + 1023) & ~1023u;
constexpr uint32_t kPKQ2 = kPKB + 16384;  // channel: second copy of the bf16 [K; Q] tile (TMA), 32 KiB
constexpr uint32_t kPStrong = kPKQ2 + 32768;  // channel: int flags [128], then per-warp lists [4][32] + counts [4]
constexpr uint32_t kPrepBytesChannel = kPStrong + 1024 + 1024;
constexpr float kStrongSpread = 14.f;  // log2 units: a larger within-chunk spread makes a channel "strong"

// TMEM columns of one prep pipeline
constexpr uint32_t kTG = 0, kTW = 64, kTU = 192, kPrepTmemCols = 256;

struct PrepArgs {
    const float* g;
    const float* beta;
    int T, H, NC;
    int* status;
    int pro;                  // gdr_prologue flags
    const float* gate_scale;  // [H] or NULL
    const float* erase;       // Gated DeltaNet-2 (EW): [B,T,H,d_k] erase gate
    const float* write;       // Gated DeltaNet-2 (EW): [B,T,H,d_v] write gate
};

// Inverse L2 norms of the 128 rows of the [K; Q] tile (prologue GDR_PRO_L2NORM_QK), fp32 [128]:
// in the slack after the scalar gate's 2^-Gamma table, or after the channel gate's strong lists.
__host__ __device__ constexpr uint32_t nrm_off(int mode) {
    return mode == GDR_DECAY_CHANNEL ? kPStrong + 1280 : kFInvE + 512;
}
static_assert(kFInvE + 512 + 512 <= kPrepBytesScalar, "norm table fits the scalar layout");
static_assert(kPStrong + 1280 + 512 <= kPrepBytesChannel, "norm table fits the channel layout");

struct PrepSmem {
    uint8_t* base;
    uint64_t* bars;  // [4]: TMA ([K; Q], and V for the channel gate), Gram, W/U, TMA of V (the
                     // channel gate: of its tile copy)
    uint32_t tmem;
    int bar_id;      // named barrier of this pipeline's 128 threads
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ uint32_t pack2h(float a, float b) {
    __half2 t = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&t);
}
__device__ __forceinline__ uint4 pack8h(const float* f) {
    return make_uint4(pack2h(f[0], f[1]), pack2h(f[2], f[3]), pack2h(f[4], f[5]), pack2h(f[6], f[7]));
}
__device__ __forceinline__ void unpack8bf(uint4 u, float* f) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __nv_bfloat162 t = *reinterpret_cast<const __nv_bfloat162*>(&w[i]);
        f[2 * i] = __low2float(t);
        f[2 * i + 1] = __high2float(t);
    }
}
__device__ __forceinline__ void unpack8h(uint4 u, float* f) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __half2 t = *reinterpret_cast<const __half2*>(&w[i]);
        f[2 * i] = __low2float(t);
        f[2 * i + 1] = __high2float(t);
    }
}
__device__ __forceinline__ void st16(void* p, uint4 v) { *reinterpret_cast<uint4*>(p) = v; }
// Eight fp32 gate values of chunk row r, columns col0 .. col0 + 7 (rows past the tail give 0).
__device__ __forceinline__ void load_gate8(const float* gate, size_t tok0, int r, int H, int n, int col0, int ld,
                                           float (&x)[8]) {
    if (r < n) {
        const float4* p = reinterpret_cast<const float4*>(gate + (tok0 + (size_t)r * H) * ld + col0);
        const float4 a = p[0], b = p[1];
        x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
        x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
    } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = 0.f;
    }
}
__device__ __forceinline__ uint4 ld16(const void* p) { return *reinterpret_cast<const uint4*>(p); }

// 16 x 16 output tile of C = A (16 x K) * B (K x 16) on warp MMAs (tf32, fp32 accumulate).
// A(row, k) and B(k, col) are read through the accessors; the result stays in fragments
// (c[nt][0..3] for the two 8-column halves).
template <typename FA, typename FB>
__device__ __forceinline__ void warp_gemm16(float (&c)[2][4], FA A, FB B, int K, int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) c[nt][e] = 0.f;
    for (int k0 = 0; k0 < K; k0 += 8) {
        const uint32_t a[4] = {to_tf32(A(g, k0 + t)), to_tf32(A(g + 8, k0 + t)), to_tf32(A(g, k0 + t + 4)),
                               to_tf32(A(g + 8, k0 + t + 4))};
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const uint32_t bb[2] = {to_tf32(B(k0 + t, nt * 8 + g)), to_tf32(B(k0 + t + 4, nt * 8 + g))};
            mma_tf32_16x8x8(c[nt], a, bb);
        }
    }
}

// Stores a 16 x 16 fragment tile (times `sign`) through the accessor dst(row, col) = value.
template <typename FD>
__device__ __forceinline__ void warp_store16(const float (&c)[2][4], FD D, float sign, int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        D(g, nt * 8 + 2 * t, sign * c[nt][0]);
        D(g, nt * 8 + 2 * t + 1, sign * c[nt][1]);
        D(g + 8, nt * 8 + 2 * t, sign * c[nt][2]);
        D(g + 8, nt * 8 + 2 * t + 1, sign * c[nt][3]);
    }
}

// T = (I + A)^-1 for the 64 x 64 strictly-lower A held transposed in sAt (sAt[i][r] = A[r][i]).
// Diagonal 16 x 16 blocks by right-looking forward substitution (one thread per column), then
// T_IJ = -T_II (A_IJ T_JJ) for the two 32 x 32 halves and -T_hi (A_ll T_lo) for the lower-left
// 32 x 32 block, on warp MMAs. The strictly upper part of sT is zero and never written.
__device__ void unit_lower_inverse64(const float* __restrict__ sAt, float* __restrict__ sT, float* __restrict__ sX,
                                     int lt, int bar_id) {
    // executed by 128 threads (4 warps); bar_id is their named barrier
    const int lw = lt >> 5, lane = lt & 31;
    auto At = [&](int r, int i) { return sAt[i * kLdA + r]; };  // A[r][i]
    if (lt < 64) {
        const int base = (lt >> 4) * 16, j = lt & 15;
        float x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) x[r] = (r == j) ? 1.f : 0.f;
#pragma unroll
        for (int i = 0; i < 15; ++i) {
            // column i of the diagonal block, A[base + r][base + i] for r = 0..15, as four 16-byte loads
            const float4* col = reinterpret_cast<const float4*>(sAt + (base + i) * kLdA + base);
            float a[16];
#pragma unroll
            for (int q4 = (i + 1) >> 2; q4 < 4; ++q4) {
                const float4 t = col[q4];
                a[4 * q4] = t.x;
                a[4 * q4 + 1] = t.y;
                a[4 * q4 + 2] = t.z;
                a[4 * q4 + 3] = t.w;
            }
#pragma unroll
            for (int r = i + 1; r < 16; ++r) x[r] = fmaf(-a[r], x[i], x[r]);
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) sT[(base + r) * kLdT + base + j] = x[r];
    }
    named_bar(bar_id, 128);
    // T_10 = -T_11 (A_10 T_00) (warp 0), T_32 = -T_33 (A_32 T_22) (warp 1)
    if (lw < 2) {
        const int I = 2 * lw + 1, J = 2 * lw;
        float* X = sX + lw * 16 * kLdX;  // 16 x 16 scratch per warp
        float c[2][4];
        warp_gemm16(c, [&](int r, int k) { return At(16 * I + r, 16 * J + k); },
                    [&](int k, int col) { return sT[(16 * J + k) * kLdT + 16 * J + col]; }, 16, lane);
        warp_store16(c, [&](int r, int col, float v) { X[r * kLdX + col] = v; }, 1.f, lane);
        __syncwarp();
        warp_gemm16(c, [&](int r, int k) { return sT[(16 * I + r) * kLdT + 16 * I + k]; },
                    [&](int k, int col) { return X[k * kLdX + col]; }, 16, lane);
        warp_store16(c, [&](int r, int col, float v) { sT[(16 * I + r) * kLdT + 16 * J + col] = v; }, -1.f, lane);
    }
    named_bar(bar_id, 128);
    // lower-left 32 x 32: Y = A_ll T_lo, then T_ll = -T_hi Y; warp w owns the 16 x 16 quadrant (qr, qc)
    {
        const int qr = lw >> 1, qc = lw & 1;
        float c[2][4];
        warp_gemm16(c, [&](int r, int k) { return At(32 + 16 * qr + r, k); },
                    [&](int k, int col) { return sT[k * kLdT + 16 * qc + col]; }, 32, lane);
        warp_store16(c, [&](int r, int col, float v) { sX[(16 * qr + r) * kLdX + 16 * qc + col] = v; }, 1.f, lane);
        named_bar(bar_id, 128);
        warp_gemm16(c, [&](int r, int k) { return sT[(32 + 16 * qr + r) * kLdT + 32 + k]; },
                    [&](int k, int col) { return sX[k * kLdX + 16 * qc + col]; }, 32, lane);
        warp_store16(c, [&](int r, int col, float v) { sT[(32 + 16 * qr + r) * kLdT + 16 * qc + col] = v; }, -1.f,
                     lane);
    }
    named_bar(bar_id, 128);
}

// One-time set-up of a prep pipeline's shared memory: the zero block under T diag(beta) (rows
// 64-127 of the M = 128 operand of the W product) and, for the channel gate, the strictly upper
// part of T (never written by the solve; the other modes clear it in each task, as T moves).
template <int MODE>
__device__ void prep_init(const PrepSmem& ps, int lt) {
    uint8_t* z = ps.base + (MODE == GDR_DECAY_CHANNEL ? kPTBZ : kFTBZ) + 8192;
    for (int i = lt; i < 512; i += kPrepThreads) reinterpret_cast<uint4*>(z)[i] = make_uint4(0, 0, 0, 0);  // 8 KiB
    if (MODE == GDR_DECAY_CHANNEL) {
        float* sT = reinterpret_cast<float*>(ps.base + kPT);
        for (int i = lt; i < 64 * kLdT; i += kPrepThreads) sT[i] = 0.f;
    }
}

// Computes the hand-off block of chunk c of head (b, h) into `out` (global memory). Executed by the
// 256 threads of one pipeline (8 warps: TMEM lane quadrant q = warp & 3, column half hf = warp >> 2);
// `it` counts the pipeline's previous tasks (mbarrier phase parity). DeltaNet and the scalar gate
// load the [K; Q] tile of the pipeline's next task (chunk nc of head (nb, nh); nc < 0: none) once
// this task's T diag(beta) is built; `pre` says that the previous task did so for this one.
template <int MODE, bool PRO, bool EW = false>
__device__ void prep_chunk(const PrepArgs& P, const CUtensorMap* mq, const CUtensorMap* mk, const CUtensorMap* mv,
                           const PrepSmem& ps, int b, int h, int c, uint8_t* __restrict__ out, uint32_t it, int lt,
                           uint32_t& n_copies, int nb, int nh, int nc, bool pre) {
    constexpr bool PF = MODE != GDR_DECAY_CHANNEL;  // alternating regions, tile of the next task ahead
    const int lw = lt >> 5, lane = lt & 31;
    const int q = lw & 3, hf = lw >> 2;
    const uint32_t par = it & 1u;
    uint8_t* sm = ps.base;
    uint8_t* sKQ = sm + (PF ? par * kFRegion : kPKQ);
    uint8_t* sAT = sm + (PF ? (par ^ 1u) * kFRegion : kPA);  // A^T, then T: the other region
    uint8_t* sV = sm + (PF ? kFV : kPV);
    uint8_t* sTB = sm + (PF ? kFTBZ : kPTBZ);
    float* sAt = reinterpret_cast<float*>(sAT);
    float* sT = reinterpret_cast<float*>(PF ? sAT + 64 * kLdA * 4 : sm + kPT);
    float* sX = reinterpret_cast<float*>(PF ? sKQ + 8192 : sm + kPX);  // PF: the first box of Q rows
    float* sBeta = reinterpret_cast<float*>(sm + (PF ? kFBeta : kPBeta));
    float* sGam = reinterpret_cast<float*>(sm + (PF ? kFGam : kPGam));
    float* sInvE = reinterpret_cast<float*>(sm + (PF ? kFInvE : kPInvE));
    uint8_t* sKB = sm + kPKB;
    uint64_t* barT = ps.bars;
    uint64_t* barG = ps.bars + 1;
    uint64_t* barW = ps.bars + 2;
    uint64_t* barV = ps.bars + 3;  // PF only (the channel gate's tile copy uses it otherwise)
    const int T = P.T, H = P.H;
    const int c0 = c * kC;
    const int n = min(kC, T - c0);
    const size_t tok0 = ((size_t)b * T + c0) * H + h;  // chunk row r is token tok0 + r * H
    // prologue steps: compiled only into the PRO instantiations, so the plain call's code is unchanged
    const bool norm = PRO && (P.pro & GDR_PRO_L2NORM_QK) != 0, gate = PRO && (P.pro & GDR_PRO_GATE_SOFTPLUS) != 0;
    float* sNrm = reinterpret_cast<float*>(sm + nrm_off(MODE));

    // ---- 1. TMA: K and Q into the two halves of the 128-row [K; Q] tile, V; beta and the
    //         cumulative log-decay (log2 units; rows past the tail repeat Gamma_{n-1}) meanwhile
    if (lt == 0) {
        bulk_wait_read<0>();  // the previous task's W / U^T bulk stores have read the K / V tiles
        uint64_t* bv = PF ? barV : barT;
        if (!(PF && pre)) {
            mbar_arrive_expect_tx(barT, (PF ? 4 : 6) * 8192);
            tma_load_4d(sKQ, mk, 0, h, c0, b, barT);
            tma_load_4d(sKQ + 16384, mk, 64, h, c0, b, barT);
            tma_load_4d(sKQ + 8192, mq, 0, h, c0, b, barT);
            tma_load_4d(sKQ + 24576, mq, 64, h, c0, b, barT);
        }
        if (PF) mbar_arrive_expect_tx(barV, 2 * 8192);
        tma_load_4d(sV, mv, 0, h, c0, b, bv);
        tma_load_4d(sV + 8192, mv, 64, h, c0, b, bv);
    }
    if (lw == 7) {
        const bool sig = PRO && (P.pro & GDR_PRO_BETA_SIGMOID) != 0;
#pragma unroll
        for (int m = 0; m < 2; ++m) {
            const int r = lane + 32 * m;
            // Gated DeltaNet-2: the gates replace beta (1 here), e in the erase operands, w in V
            float x = (r < n) ? (EW ? 1.f : P.beta[tok0 + (size_t)r * H]) : 0.f;
            if (sig && r < n) x = pro_sigmoid(x);
            sBeta[r] = x;
        }
    }
    const float A = (gate && P.gate_scale != nullptr) ? P.gate_scale[h] : 1.f;
    if (MODE == GDR_DECAY_SCALAR) {
        if (lw == 6) {
            float x0 = (lane < n) ? P.g[tok0 + (size_t)lane * H] : 0.f;
            float x1 = (lane + 32 < n) ? P.g[tok0 + (size_t)(lane + 32) * H] : 0.f;
            if (gate) {
                x0 = (lane < n) ? pro_gate(x0, A) : 0.f;
                x1 = (lane + 32 < n) ? pro_gate(x1, A) : 0.f;
            }
            x0 *= kLog2e;
            x1 *= kLog2e;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float y0 = __shfl_up_sync(0xffffffffu, x0, off);
                const float y1 = __shfl_up_sync(0xffffffffu, x1, off);
                if (lane >= off) {
                    x0 += y0;
                    x1 += y1;
                }
            }
            x1 += __shfl_sync(0xffffffffu, x0, 31);
            sGam[lane] = x0;
            sGam[lane + 32] = x1;
            // pairwise decays 2^(Gamma_r - Gamma_i) as 2^Gamma_r * 2^-Gamma_i when every |Gamma| stays
            // well inside the normal fp32 exponent range (both factors finite and normal)
            sInvE[lane] = fast_exp2(-x0);
            sInvE[lane + 32] = fast_exp2(-x1);
            const bool fac = __all_sync(0xffffffffu, fabsf(x0) <= 120.f && fabsf(x1) <= 120.f);
            if (lane == 0) *reinterpret_cast<int*>(sInvE + 64) = fac ? 1 : 0;
        }
    } else if (MODE == GDR_DECAY_CHANNEL) {
        if (lt < kD) {
            float gv[kC];
#pragma unroll
            for (int r = 0; r < kC; ++r) gv[r] = (r < n) ? P.g[(tok0 + (size_t)r * H) * kD + lt] : 0.f;
            if (gate) {
#pragma unroll
                for (int r = 0; r < kC; ++r) gv[r] = (r < n) ? pro_gate(gv[r], A) : 0.f;
            }
            float acc = 0.f, lo = 0.f, hi = 0.f;
#pragma unroll
            for (int r = 0; r < kC; ++r) {
                acc = fmaf(gv[r], kLog2e, acc);
                sGam[r * kD + lt] = acc;
                lo = fminf(lo, acc);
                hi = fmaxf(hi, acc);
            }
            // a channel whose cumulative log-decay spreads wider than kStrongSpread inside the chunk
            // stays out of the factored tensor-core product (its factors could leave fp16's range)
            const bool strong = hi - lo > kStrongSpread;
            int* sStrong = reinterpret_cast<int*>(sm + kPStrong);
            sStrong[lt] = strong ? 1 : 0;
            const unsigned m = __ballot_sync(0xffffffffu, strong);
            if (strong) sStrong[128 + 32 * lw + __popc(m & ((1u << lane) - 1u))] = lt;
            if (lane == 0) sStrong[256 + lw] = __popc(m);
        }
    }
    named_bar(ps.bar_id, kPrepThreads);
    // channel gate: the number of strong channels in this chunk; if any, a second copy of the bf16 K
    // and Q tiles (which step 2 overwrites) for their exact terms and for K*gamma
    int n_strong = 0;
    uint64_t* barT2 = ps.bars + 3;
    if (MODE == GDR_DECAY_CHANNEL) {
        const int* sStrong = reinterpret_cast<const int*>(sm + kPStrong);
        n_strong = sStrong[256] + sStrong[257] + sStrong[258] + sStrong[259];
        if (n_strong > 0 && lt == 0) {
            uint8_t* sKQ2 = sm + kPKQ2;
            mbar_arrive_expect_tx(barT2, 4 * 8192);
            tma_load_4d(sKQ2, mk, 0, h, c0, b, barT2);
            tma_load_4d(sKQ2 + 16384, mk, 64, h, c0, b, barT2);
            tma_load_4d(sKQ2 + 8192, mq, 0, h, c0, b, barT2);
            tma_load_4d(sKQ2 + 24576, mq, 64, h, c0, b, barT2);
        }
    }
    mbar_wait(barT, par, P.status);
    const uint32_t tG = ps.tmem + kTG, tW = ps.tmem + kTW, tU = ps.tmem + kTU;
    // Gram products for the scalar gate / DeltaNet straight from the bf16 tiles (a prologue's norms
    // rescale them in the epilogue). Issued here rather than before the barrier above: measured
    // slower there, as the other warps then wait for the issue.
    if (PF && lt == 0) {
        tc_fence_after();
        const uint32_t id = idesc_bf16(128, 64, false, false);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            const uint64_t d = sdesc(smem_u32(sKQ) + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
            mma_f16(tG, d, d, id, ks > 0);  // B = the K rows (first 64 rows) of the same tile
        }
        mma_commit(barG);
    }
    if (norm) {
        // inverse L2 norms of the 128 tile rows (K rows 0-63, Q rows 64-127; rows past the tail are
        // zero and get 0), two threads per row; the Gram products below run on the raw tiles and
        // are rescaled in their epilogue
        const int row = lt >> 1, half = lt & 1;
        float ss = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            float f[8];
            unpack8bf(ld16(sKQ + kmajor_off(row, 64 * half + 8 * j, 128)), f);
#pragma unroll
            for (int e = 0; e < 8; ++e) ss = fmaf(f[e], f[e], ss);
        }
        ss += __shfl_xor_sync(0xffffffffu, ss, 1);
        if (half == 0) sNrm[row] = pro_inv_norm(ss);
        named_bar(ps.bar_id, kPrepThreads);
    }

    // ---- 2. Q*gamma and K*gamma_C/gamma hand-off images; channel gate: decay-factored Gram operands
    const int ref = (n - 1) >> 1;
    // channel gate: strong flags of this thread's 8 columns (the same in each of its 4 tasks)
    bool weak8[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) weak8[e] = true;
    if (MODE == GDR_DECAY_CHANNEL && n_strong > 0) {
        const int* fl = reinterpret_cast<const int*>(sm + kPStrong) + (lt & 15) * 8;
#pragma unroll
        for (int e = 0; e < 8; ++e) weak8[e] = fl[e] == 0;
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int task = lt + kPrepThreads * j;
        const int r = task >> 4, col0 = (task & 15) * 8;
        const uint32_t okr = kmajor_off(r, col0, 128), oqr = kmajor_off(kC + r, col0, 128);
        float kx[8], qx[8];
        unpack8bf(ld16(sKQ + okr), kx);
        unpack8bf(ld16(sKQ + oqr), qx);
        if (norm) {
            const float nk = sNrm[r], nq = sNrm[kC + r];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                kx[e] *= nk;
                qx[e] *= nq;
            }
        }
        float qg[8], kt[8];
        if (MODE == GDR_DECAY_NONE) {
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                qg[e] = qx[e];
                kt[e] = kx[e];
            }
        } else if (MODE == GDR_DECAY_SCALAR) {
            const float fr = fast_exp2(sGam[r]), ft = fast_exp2(sGam[kC - 1] - sGam[r]);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                qg[e] = qx[e] * fr;
                kt[e] = kx[e] * ft;
            }
        } else {
            float ka[8], qa[8], kb[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float G = sGam[r * kD + col0 + e];
                const float Gr = sGam[ref * kD + col0 + e];
                const float GC = sGam[(kC - 1) * kD + col0 + e];
                // factors within 2^kStrongSpread; a strong channel's terms are added on the CUDA cores
                const float up = weak8[e] ? fast_exp2(G - Gr) : 0.f, dn = weak8[e] ? fast_exp2(Gr - G) : 0.f;
                qg[e] = qx[e] * fast_exp2(G);
                kt[e] = kx[e] * fast_exp2(GC - G);
                ka[e] = kx[e] * up;
                qa[e] = qx[e] * up;
                kb[e] = kx[e] * dn;
            }
            if (EW) {  // the erase direction e (.) k on the left of the Gram (and in K*gamma for W)
                float er[8];
                load_gate8(P.erase, tok0, r, H, n, col0, kD, er);
#pragma unroll
                for (int e = 0; e < 8; ++e) ka[e] *= er[e];
            }
            st16(sKQ + okr, pack8h(ka));
            st16(sKQ + oqr, pack8h(qa));
            st16(sKB + kmajor_off(r, col0, 64), pack8h(kb));
        }
        st16(out + kOffWQ + oqr, pack8h(qg));
        st16(out + kOffKT + mnmajor_off(r, col0, 64), pack8h(kt));
    }
    if (lt < kD) {
        float gc = 1.f;
        if (MODE == GDR_DECAY_SCALAR) gc = fast_exp2(sGam[kC - 1]);
        if (MODE == GDR_DECAY_CHANNEL) gc = fast_exp2(sGam[(kC - 1) * kD + lt]);
        reinterpret_cast<float*>(out + kOffGam)[lt] = gc;
    }
    if (MODE == GDR_DECAY_CHANNEL) {
        fence_proxy_async_smem();
        tc_fence_before();
        named_bar(ps.bar_id, kPrepThreads);
        tc_fence_after();
        if (lt == 0) {
            const uint32_t id = idesc_f16(128, 64, false, false);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                mma_f16(tG, sdesc(smem_u32(sKQ) + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024),
                        sdesc(smem_u32(sKB) + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024), id, ks > 0);
            mma_commit(barG);
        }
    }
    __syncwarp();
    mbar_wait(barG, par, P.status);
    tc_fence_after();

    // ---- 3. A (strictly lower, beta_r folded in; stored transposed) and P (causal incl. diagonal):
    //         thread (q, hf) takes TMEM lane 32 q + lane (K rows for q < 2, Q rows for q >= 2),
    //         columns i in [32 hf, 32 hf + 32)
    {
        const int rr = (q & 1) * 32 + lane;
        float x[32];
        tmem_ld32(tG + ((uint32_t)(q * 32) << 16) + 32 * hf, x);
        float d[32];
        if (MODE == GDR_DECAY_SCALAR) {
            const float G2r = sGam[rr];
            if (*reinterpret_cast<const int*>(sInvE + 64)) {  // one exponential per thread
                const float er = fast_exp2(G2r);
#pragma unroll
                for (int e = 0; e < 32; ++e) d[e] = er * sInvE[32 * hf + e];
            } else {
#pragma unroll
                for (int e = 0; e < 32; ++e) d[e] = fast_exp2(fminf(G2r - sGam[32 * hf + e], 0.f));
            }
        }
        const float br = sBeta[rr];
        tmem_ld_wait();
        if (MODE != GDR_DECAY_CHANNEL && norm) {  // the Gram of the raw tiles, rescaled
            const float nr = sNrm[q * 32 + lane];
#pragma unroll
            for (int e = 0; e < 32; ++e) x[e] *= nr * sNrm[32 * hf + e];
        }
        if (MODE == GDR_DECAY_CHANNEL && n_strong > 0) {
            // the strong channels' terms, left out of the tensor-core product: k_r,d k_i,d
            // 2^(Gamma_r,d - Gamma_i,d) (or q_r,d ...) from the bf16 copy of the tiles, fp32
            mbar_wait(barT2, n_copies & 1u, P.status);
            const int* sStrong = reinterpret_cast<const int*>(sm + kPStrong);
            const uint8_t* sKQ2 = sm + kPKQ2;
            const int row = q * 32 + lane;  // tile row: K rows 0-63, Q rows 64-127
#pragma unroll 1
            for (int w4 = 0; w4 < 4; ++w4) {
                const int cnt = sStrong[256 + w4];
#pragma unroll 1
                for (int kk = 0; kk < cnt; ++kk) {
                    const int dch = sStrong[128 + 32 * w4 + kk];
                    float a = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(
                                  sKQ2 + kmajor_off(row, dch, 128))) * (norm ? sNrm[row] : 1.f);
                    if (EW && row < kC) a *= (row < n) ? P.erase[(tok0 + (size_t)row * H) * kD + dch] : 0.f;
                    const float Gr = sGam[rr * kD + dch];
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const int i = 32 * hf + e;
                        const float ki = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(
                                             sKQ2 + kmajor_off(i, dch, 128))) * (norm ? sNrm[i] : 1.f);
                        const float f = (i <= rr) ? fast_exp2(Gr - sGam[i * kD + dch]) : 0.f;
                        x[e] = fmaf(a * ki, f, x[e]);
                    }
                }
            }
        }
        if (q < 2) {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const int i = 32 * hf + e;
                float a = (i < rr && rr < n) ? br * x[e] : 0.f;
                if (MODE == GDR_DECAY_SCALAR) a *= d[e];
                sAt[i * kLdA + rr] = a;
            }
        } else {
            float p[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const int i = 32 * hf + e;
                float v = (i <= rr && rr < n) ? x[e] : 0.f;
                if (MODE == GDR_DECAY_SCALAR) v *= d[e];
                p[e] = v;
            }
#pragma unroll
            for (int ci = 0; ci < 4; ++ci) st16(out + kOffP + kmajor_off(rr, 32 * hf + ci * 8, 64), pack8h(p + ci * 8));
        }
    }
    if (PF) {
        // the strictly upper blocks of T that the solve never writes (T_01, T_23 and the upper-right
        // 32 x 32) but reads or scales: this region held a tile
#pragma unroll
        for (int j = 0; j < 6; ++j) {
            const int i = lt + kPrepThreads * j;
            const int r = i < 256 ? i >> 4 : i < 512 ? 32 + ((i - 256) >> 4) : (i - 512) >> 5;
            const int col = i < 256 ? 16 + (i & 15) : i < 512 ? 48 + (i & 15) : 32 + (i & 31);
            sT[r * kLdT + col] = 0.f;
        }
    }
    tc_fence_before();
    named_bar(ps.bar_id, kPrepThreads);

    // ---- 4. warps 0-3: UT transform T = (I + A)^-1;  warps 4-7: K*gamma (in place over the K rows)
    //         and V as fp16 operands of the W / U MMAs
    if (lw < 4) {
        unit_lower_inverse64(sAt, sT, sX, lt, ps.bar_id + 1);
    } else {
        const int lt4 = lt - 128;
        if (PF) mbar_wait(barV, par, P.status);
#pragma unroll 4
        for (int j = 0; j < 16; ++j) {
            const int task = lt4 + 128 * j;
            const bool isv = task >= 1024;
            const int r = (task & 1023) >> 4, col0 = (task & 15) * 8;
            uint8_t* p = isv ? sV + kmajor_off(r, col0, 64) : sKQ + kmajor_off(r, col0, 128);
            float x[8];
            if (!isv && MODE == GDR_DECAY_CHANNEL) {
                // K' = K 2^(Gamma - Gamma_ref) times 2^Gamma_ref gives K*gamma on the other channels; a
                // strong channel's K' is zero, its K*gamma comes from the bf16 copy (every factor <= 1)
                unpack8h(ld16(p), x);
                if (n_strong > 0) {
                    const int* fl = reinterpret_cast<const int*>(sm + kPStrong) + col0;
                    float kc[8];
                    unpack8bf(ld16(sm + kPKQ2 + kmajor_off(r, col0, 128)), kc);
                    const float nk = norm ? sNrm[r] : 1.f;
                    if (EW) {
                        float er[8];
                        load_gate8(P.erase, tok0, r, H, n, col0, kD, er);
#pragma unroll
                        for (int e = 0; e < 8; ++e) kc[e] *= er[e];
                    }
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        x[e] = fl[e] ? kc[e] * nk * fast_exp2(sGam[r * kD + col0 + e])
                                     : x[e] * fast_exp2(sGam[ref * kD + col0 + e]);
                } else {
#pragma unroll
                    for (int e = 0; e < 8; ++e) x[e] *= fast_exp2(sGam[ref * kD + col0 + e]);
                }
            } else {
                unpack8bf(ld16(p), x);
                if (EW && isv) {  // the gated write target w (.) v
                    float wr[8];
                    load_gate8(P.write, tok0, r, H, n, col0, kD, wr);
#pragma unroll
                    for (int e = 0; e < 8; ++e) x[e] *= wr[e];
                }
                if (!isv && (MODE == GDR_DECAY_SCALAR || norm)) {
                    float fr = MODE == GDR_DECAY_SCALAR ? fast_exp2(sGam[r]) : 1.f;
                    if (norm) fr *= sNrm[r];
#pragma unroll
                    for (int e = 0; e < 8; ++e) x[e] *= fr;
                }
            }
            st16(p, pack8h(x));
        }
    }
    named_bar(ps.bar_id, kPrepThreads);
    // T diag(beta) as fp16
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const int task = lt + kPrepThreads * j;
        const int r = task >> 3, i0 = (task & 7) * 8;
        float t8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) t8[e] = sT[r * kLdT + i0 + e] * sBeta[i0 + e];
        st16(sTB + kmajor_off(r, i0, 64), pack8h(t8));
    }
    fence_proxy_async_smem();
    tc_fence_before();
    named_bar(ps.bar_id, kPrepThreads);
    tc_fence_after();

    // ---- 5. W = [T diag(beta); 0] (K*gamma) (M = 128, N = 128) and U^T = V^T (T diag(beta))^T (M = 128, N = 64)
    if (lt == 0) {
        const uint32_t idW = idesc_f16(128, 128, false, true);
        const uint32_t idU = idesc_f16(128, 64, true, false);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            const uint64_t tb = sdesc(smem_u32(sTB) + ks * 32, 16, 1024);
            mma_f16(tW, tb, sdesc(smem_u32(sKQ) + ks * 2048, 16384, 1024), idW, ks > 0);
            mma_f16(tU, sdesc(smem_u32(sV) + ks * 2048, 8192, 1024), tb, idU, ks > 0);
        }
        mma_commit(barW);
        if (PF && nc >= 0) {
            // the next task's [K; Q] tile into the region of A^T and T, which no one reads any more
            // (every thread's accesses were ordered before the async proxy ahead of the last barrier)
            const int nc0 = nc * kC;
            mbar_arrive_expect_tx(barT, 4 * 8192);
            tma_load_4d(sAT, mk, 0, nh, nc0, nb, barT);
            tma_load_4d(sAT + 16384, mk, 64, nh, nc0, nb, barT);
            tma_load_4d(sAT + 8192, mq, 0, nh, nc0, nb, barT);
            tma_load_4d(sAT + 24576, mq, 64, nh, nc0, nb, barT);
        }
    }
    __syncwarp();
    mbar_wait(barW, par, P.status);
    tc_fence_after();
    // ---- 6. W rows and U^T rows to staging images (the K / V tiles are free now), bulk-stored out
    {
        uint8_t* stW = sKQ;  // W rows 0-63 in the 128-row K-major layout of the [W; Q*gamma] image
        uint8_t* stU = sV;   // U^T, 128-row K-major (one 64-column block)
        const uint32_t loff = (uint32_t)(q * 32) << 16;
        const int row = q * 32 + lane;
        if (q < 2) {
#pragma unroll
            for (int q2 = 0; q2 < 2; ++q2) {
                float x[32];
                tmem_ld32(tW + loff + 64 * hf + 32 * q2, x);
                tmem_ld_wait();
#pragma unroll
                for (int ci = 0; ci < 4; ++ci)
                    st16(stW + kmajor_off(row, 64 * hf + 32 * q2 + ci * 8, 128), pack8h(x + ci * 8));
            }
        }
        float x[32];
        tmem_ld32(tU + loff + 32 * hf, x);
        tmem_ld_wait();
#pragma unroll
        for (int ci = 0; ci < 4; ++ci) st16(stU + kmajor_off(row, 32 * hf + ci * 8, 128), pack8h(x + ci * 8));
        fence_proxy_async_smem();
        tc_fence_before();
        named_bar(ps.bar_id, kPrepThreads);
        if (MODE == GDR_DECAY_CHANNEL && n_strong > 0) ++n_copies;
        if (lt == 0) {  // the next task waits for these reads before its TMA loads into the same tiles
            bulk_s2g(out + kOffWQ, stW, 8192);
            bulk_s2g(out + kOffWQ + 16384, stW + 16384, 8192);
            bulk_s2g(out + kOffUT, stU, 16384);
            bulk_commit();
        }
    }
}

// Standalone prep kernel: one pipeline per CTA, persistent over the chunk tasks t = blockIdx.x,
// blockIdx.x + gridDim.x, ... for the first NCp chunks of every head (t = (b * H + h) * NCp + c, the
// block's index in the workspace; NCp = NC on the two-pass path, the fused kernel's c1 before it).
// At the start of each task the tiles of the CTA's next task are prefetched into L2; for DeltaNet
// and the scalar gate its [K; Q] tile then comes into shared memory during this task's W / U
// products (prep kernel 241 -> 238 us at B16 H8 T4096). The scalar and DeltaNet variants run at 96
// registers per thread (no spills; measured 1-2.5 % faster than the 128 two CTAs per SM would allow).
template <int MODE, bool PRO, bool EW = false>
__global__ void __maxnreg__(MODE == GDR_DECAY_CHANNEL ? 240 : 96)
chunk_prep_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
                  const __grid_constant__ CUtensorMap mv, PrepArgs P, uint8_t* __restrict__ ws, int NCp, int n_tasks) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t bars[4];
    __shared__ uint32_t tmem_base;
    const int lt = threadIdx.x;
    if (lt == 0) {
        for (int i = 0; i < 4; ++i) mbar_init(&bars[i], 1);
        fence_mbar_init();
    }
    if (lt < 32) {
        tmem_alloc(&tmem_base, kPrepTmemCols);
        tmem_relinquish();
    }
    PrepSmem ps{align1024(smem_raw), bars, 0, 1};
    prep_init<MODE>(ps, lt);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    ps.tmem = tmem_base;
    uint32_t it = 0, n_copies = 0;  // tasks so far; channel-gate tile copies so far (mbarrier parities)
    for (int t = blockIdx.x; t < n_tasks; t += gridDim.x, ++it) {
        const int c = t % NCp, bh = t / NCp;
        const int h = bh % P.H, b = bh / P.H;
        const int tn = t + gridDim.x;
        if (lt == 0 && tn < n_tasks) {
            const int cn = tn % NCp, bhn = tn / NCp;
            const int hn = bhn % P.H, bn = bhn / P.H;
            tma_prefetch_l2_4d(&mk, 0, hn, cn * kC, bn);
            tma_prefetch_l2_4d(&mk, 64, hn, cn * kC, bn);
            tma_prefetch_l2_4d(&mq, 0, hn, cn * kC, bn);
            tma_prefetch_l2_4d(&mq, 64, hn, cn * kC, bn);
            tma_prefetch_l2_4d(&mv, 0, hn, cn * kC, bn);
            tma_prefetch_l2_4d(&mv, 64, hn, cn * kC, bn);
        }
        uint8_t* out = ws + (size_t)t * kHandoffStride;
        const int cn = tn % NCp, bhn = tn / NCp;
        prep_chunk<MODE, PRO, EW>(P, &mq, &mk, &mv, ps, b, h, c, out, it, lt, n_copies, bhn / P.H, bhn % P.H,
                                  tn < n_tasks ? cn : -1, it > 0);
    }
    if (lt == 0) bulk_wait<0>();
    tc_fence_before();
    __syncthreads();
    if (lt < 32) tmem_dealloc(tmem_base, kPrepTmemCols);
}

// ------------------------------------------------------------------- state pass --
// One CTA per (b, h): 16 epilogue warps (warp w reads TMEM lane quadrant w & 3 and column group
// w >> 2), one issuer warp (MMAs, output stores) and one copy warp (bulk copies of the hand-off
// blocks, ring flags). The fp32 state is the TMEM accumulator of the state product; its fp16 copy
// and Delta^T live in TMEM as the A operands of the MMAs, so the S-dependent products read only
// their B operands from shared memory. Epilogue warps hand over to the issuer through mbarriers
// (one arrival per warp).
constexpr int kEpiWarps = 16;
constexpr int kStateThreads = (kEpiWarps + 2) * 32;  // + MMA issuer warp + copy warp
constexpr uint32_t kSStageA0 = 0;
constexpr uint32_t kSStageA1 = 58368;
constexpr uint32_t kSUT0 = 116736;      // U^T stages (double-buffered, 16 KiB each)
constexpr uint32_t kSUT1 = 133120;
constexpr uint32_t kSO0 = 149504;       // output staging, double-buffered: 4 (fp32) or 2 (bf16) TMA boxes
constexpr uint32_t kSO1 = 182272;       //   of 64 rows x 128 B each
constexpr uint32_t kStateSmem = kSO1 + 32768 + 1024;
// TMEM: D1 double-buffered (corr^T | O^T, 128 columns each), D3 (the fp32 state), the fp16 state
// copy (128 x 128 -> 64 columns) and Delta^T (128 x 64 fp16 -> 32 columns)
constexpr uint32_t kTD1 = 0, kTD3 = 256, kTS = 384, kTDelta = 448, kStateTmemCols = 512;

struct StateArgs {
    const float* S0;
    float* S_T;
    int T, H, NC;
    float scale;
    int* status;
    // Segment scan: CTAs bh >= n_data run the transition chain of head bh - n_data over the same
    // hand-off blocks (identity initial state, U taken as zero), writing their state to S_T2.
    int n_data;
    float* S_T2;
};

// Where the state pass finds hand-off block c of its head, when that block is complete, and how it
// tells the producer that the block has been copied out.
struct WorkspaceSource {  // two passes: every block was written before the state pass started
    const uint8_t* base;  // block 0 of this head
    size_t cstep;         // bytes from block c to block c + 1
    __device__ const uint8_t* block(int c) const { return base + (size_t)c * cstep; }
    __device__ bool wait_ready(int, int*, volatile int*) const { return true; }
    __device__ void release(int) const {}
};

constexpr int kRing = 8;  // ring slots per head in the fused kernel when no chunk is pre-computed
struct RingSource {       // fused kernel: chunks c < c1 were written to `pre` by a prep kernel launched
                          // before; the others pass through `depth` slots, flagged by the producers
    const uint8_t* pre;   // block of chunk 0 of this head among the pre-computed ones (c1 per head)
    const uint8_t* base;  // slot 0 of this head
    const int* ready;     // [depth]: c + 1 once the block of chunk c in that slot is complete
    int* consumed;        // number of this head's chunks already copied out of the ring (counted from 0)
    int c1, depth;
    __device__ const uint8_t* block(int c) const {
        return c < c1 ? pre + (size_t)c * kHandoffStride : base + (size_t)(c % depth) * kHandoffStride;
    }
    __device__ bool wait_ready(int c, int* status, volatile int* abort) const {
        if (c < c1) return true;
        if (!flag_wait_geq(ready + c % depth, c + 1, status, abort, 128)) return false;
        fence_proxy_async_global();  // the bulk copies that follow read what the acquire made visible
        return true;
    }
    __device__ void release(int c) const {
        if (c >= c1) st_release_gpu(consumed, c + 1);
    }
};

// The state pass of one head (b, h) = bh, executed by all kStateThreads threads of the CTA, with
// kStateTmemCols TMEM columns at tbase and kStateSmem bytes of shared memory at sm (1024-aligned).
// Walks the chunks in order, reading hand-off block c through `src`.
template <typename Tout, typename Src>
__device__ void state_body(const CUtensorMap* mo, const StateArgs& A, int bh, const Src& src, uint8_t* sm,
                           uint32_t tbase, volatile int* abort, bool tr = false) {
    auto stageA = [sm](int i) { return sm + kSStageA0 + i * (kSStageA1 - kSStageA0); };  // part A stage i
    auto sUT = [sm](int i) { return sm + kSUT0 + i * (kSUT1 - kSUT0); };  // U^T stage i
    auto sO = [sm](int i) { return sm + kSO0 + i * (kSO1 - kSO0); };  // output staging buffer i
    // fullWQ/fullR/fullU: bulk copies of [W; Q*gamma], of the rest of part A and of U^T landed.
    // barA/barB/barC: MMA groups done; rFree[s]: every MMA reading stage s is done. deltaReady/
    // sReady/oStaged: all epilogue warps wrote Delta^T / the fp16 state (TMEM) / the output
    // staging (shared). oFree[b]: the output staging buffer b has been read by its store.
    // drain: last MMAs complete.
    __shared__ uint64_t fullWQ[2], fullR[2], fullU[2], barA[2], rFree[2], barB, barC, deltaReady, sReady, oStaged,
        oFree[2], drain;

    const int b = bh / A.H, h = bh % A.H;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int NC = A.NC;
    constexpr int kOutBoxes = sizeof(Tout) == 4 ? 4 : 2;
    constexpr int kOutBoxCols = 128 / kOutBoxes;
    auto wait = [&](uint64_t* bar, uint32_t parity) { return mbar_wait_abort(bar, parity, A.status, abort); };

    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&fullWQ[i], 1);
            mbar_init(&fullR[i], 1);
            mbar_init(&fullU[i], 1);
            mbar_init(&barA[i], 1);
            mbar_init(&rFree[i], 1);
            mbar_init(&oFree[i], 1);
        }
        mbar_init(&barB, 1);
        mbar_init(&barC, 1);
        mbar_init(&drain, 1);
        mbar_init(&deltaReady, kEpiWarps);
        mbar_init(&sReady, kEpiWarps);
        mbar_init(&oStaged, kEpiWarps);
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == kEpiWarps + 1) {
        // --------------------------------------------------------------- copy warp --
        // Brings hand-off blocks into shared memory (part A and U^T double-buffered) as soon as both
        // the block is ready and its buffer is free, and hands each ring slot back once all of its
        // chunk is in shared memory: all flag traffic stays off the MMA issuer's path. Chunk c + 2
        // comes in three pieces: U^T and [W; Q*gamma] once chunk c's Delta is done (their readers:
        // the epilogue warps, chunk c's first product), the rest once chunk c's last product is done.
        if (lane == 0) {
            int lastWQ[2] = {-1, -1}, lastR[2] = {-1, -1}, lastU[2] = {-1, -1};  // last chunk copied
            auto copy_wq = [&](int c) {
                mbar_arrive_expect_tx(&fullWQ[c & 1], kPartWQ);
                bulk_g2s(stageA(c & 1), src.block(c), kPartWQ, &fullWQ[c & 1]);
                lastWQ[c & 1] = c;
            };
            auto copy_r = [&](int c) {
                mbar_arrive_expect_tx(&fullR[c & 1], kPartA - kPartWQ);
                bulk_g2s(stageA(c & 1) + kPartWQ, src.block(c) + kPartWQ, kPartA - kPartWQ, &fullR[c & 1]);
                lastR[c & 1] = c;
            };
            auto copy_u = [&](int c) {
                mbar_arrive_expect_tx(&fullU[c & 1], 16384);
                bulk_g2s(sUT(c & 1), src.block(c) + kOffUT, 16384, &fullU[c & 1]);
                lastU[c & 1] = c;
            };
            bool ok = true;
            for (int st = 0; st < 2 && st < NC && ok; ++st) {
                if (!(ok = src.wait_ready(st, A.status, abort))) break;
                copy_u(st);
                copy_wq(st);
                copy_r(st);
            }
            for (int c = 0; ok && c < NC; ++c) {
                const int sb = c & 1;
                // every epilogue warp has read U^T of chunk c (and waited for it), so all of chunk c
                // is in shared memory: the ring slot goes back
                if (!wait(&deltaReady, c & 1)) break;
                src.release(c);
                if (c + 2 < NC) {
                    // chunk c's first product (barA, complete before deltaReady) has read [W; Q*gamma]
                    // of stage sb; the rest follows once every MMA of chunk c is done (gamma_C was
                    // read before deltaReady)
                    if (!wait(&barA[sb], (c >> 1) & 1)) break;
                    if (!src.wait_ready(c + 2, A.status, abort)) break;
                    copy_u(c + 2);
                    copy_wq(c + 2);
                    if (!wait(&rFree[sb], (c >> 1) & 1)) break;
                    copy_r(c + 2);
                }
            }
            // every copy issued lands before shared memory is released
            for (int sb = 0; sb < 2; ++sb) {
                if (lastWQ[sb] >= 0) mbar_wait(&fullWQ[sb], (lastWQ[sb] >> 1) & 1, A.status);
                if (lastR[sb] >= 0) mbar_wait(&fullR[sb], (lastR[sb] >> 1) & 1, A.status);
                if (lastU[sb] >= 0) mbar_wait(&fullU[sb], (lastU[sb] >> 1) & 1, A.status);
            }
        }
        __syncwarp();
    } else if (warp == kEpiWarps) {
        // ------------------------------------------------------------- issuer warp --
        if (lane == 0) {
            const uint32_t idA = idesc_f16(128, 128, false, false);
            const uint32_t idC = idesc_f16(128, 128, false, true);
            const uint32_t idB = idesc_f16(128, 64, false, false);
            int c = 0;
            for (; c < NC; ++c) {
                const int sb = c & 1;
                const uint8_t* st = stageA(sb);
                const uint32_t tD1 = tbase + kTD1 + sb * 128;
                // D1[sb] = S [W; Q*gamma]^T (M = 128, N = 128, K = 128), once the fp16 state is in TMEM
                // (one N = 128 product: a tcgen05 MMA step costs the same for N = 64 and N = 128)
                if (!wait(&sReady, c & 1) || !wait(&fullWQ[sb], (c >> 1) & 1)) break;
                tc_fence_after();
                const uint64_t dWQ = sdesc(smem_u32(st + kOffWQ), 16, 1024);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_f16_ts(tD1, tbase + kTS + ks * 8, dWQ + (uint64_t)(((ks >> 2) * 16384 + (ks & 3) * 32) >> 4),
                               idA, ks > 0);
                mma_commit(&barA[sb]);
                // output of chunk c-1 (staged by the epilogue warps in sO[(c-1)&1])
                if (c > 0) {
                    if (!wait(&oStaged, (c - 1) & 1)) break;
                    const uint8_t* so = sO((c - 1) & 1);
                    for (int bx = 0; bx < kOutBoxes; ++bx)
                        tma_store_4d(mo, so + bx * 8192, bx * kOutBoxCols, h, (c - 1) * kC, b);
                    bulk_commit();
                    bulk_wait_read<1>();  // the store of chunk c-2 has read sO[c & 1]
                    mbar_arrive(&oFree[c & 1]);
                } else {
                    mbar_arrive(&oFree[0]);
                }
                // D3 = Delta^T K~ (N = 128) and D1[sb][:, 64:128] += Delta^T P^T (N = 64)
                if (!wait(&deltaReady, c & 1) || !wait(&fullR[sb], (c >> 1) & 1)) break;
                tc_fence_after();
                const uint64_t dKT = sdesc(smem_u32(st + kOffKT), 8192, 1024);
                const uint64_t dP = sdesc(smem_u32(st + kOffP), 16, 1024);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)  // accumulates onto gamma_C * S, which D3 holds
                    mma_f16_ts(tbase + kTD3, tbase + kTDelta + ks * 8, dKT + (uint64_t)(ks * 2048 >> 4), idC, true);
                mma_commit(&barC);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_f16_ts(tD1 + 64, tbase + kTDelta + ks * 8, dP + (uint64_t)(ks * 32 >> 4), idB, true);
                mma_commit(&barB);
                if (c + 2 < NC) mma_commit(&rFree[sb]);  // stage sb may take chunk c + 2
            }
            if (c == NC && wait(&oStaged, (NC - 1) & 1)) {  // output of the last chunk
                const uint8_t* so = sO((NC - 1) & 1);
                for (int bx = 0; bx < kOutBoxes; ++bx)
                    tma_store_4d(mo, so + bx * 8192, bx * kOutBoxCols, h, (NC - 1) * kC, b);
                bulk_commit();
            }
            bulk_wait<0>();
            mma_commit(&drain);
            mbar_wait(&drain, 0, A.status);
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------- epilogue warps --
        // The fp32 state lives in TMEM (D3): each chunk's Delta^T K~ product accumulates onto
        // gamma_C * S there. After that product the epilogue warps read S once and hand its fp16
        // copy to the next chunk's MMAs; they stage the chunk's output and write gamma_C(next) * S
        // back into D3 while the next chunk's first product runs, off the chain from one chunk's
        // products to the next.
        const int quad = warp & 3, cg = warp >> 2;
        const int j = quad * 32 + lane;  // state row (d_v index) = TMEM lane
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const uint32_t tD3 = tbase + kTD3 + lane_off + 32 * cg;  // S[j][32 cg .. 32 cg + 31]
        const uint32_t tS = tbase + kTS + lane_off + 16 * cg;    // their fp16 copy
        // S_c (this thread's 32 columns, in x) becomes the fp16 operand of chunk c's MMAs
        auto hand_over = [&](const float (&x)[32]) {
            uint32_t w[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) w[e] = pack2h(x[2 * e], x[2 * e + 1]);
            tmem_st16(tS, w);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sReady);
        };
        // D3 <- gamma_C(c) * S_c, which the state product of chunk c accumulates onto; the store
        // completes before this thread's Delta hand-off of chunk c (tmem_st_wait there)
        auto decay = [&](float (&x)[32], int c) -> bool {
            if (!wait(&fullR[c & 1], (c >> 1) & 1)) return false;
            const float4* gam = reinterpret_cast<const float4*>(stageA(c & 1) + kOffGam) + 8 * cg;
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4) {
                const float4 g = gam[q4];
                x[4 * q4] *= g.x;
                x[4 * q4 + 1] *= g.y;
                x[4 * q4 + 2] *= g.z;
                x[4 * q4 + 3] *= g.w;
            }
            tmem_st32(tD3, x);
            return true;
        };
        // output staging: this thread's element of row r sits at ob + r * 128 + ((och ^ (r & 7)) << 4)
        // (128-byte swizzled TMA boxes of 64 rows); rows r = 16 cg + e, and 16 cg is a multiple of 8
        const uint32_t ob = (uint32_t)(16 * cg) * 128u +
                            (sizeof(Tout) == 4 ? (uint32_t)(j >> 5) * 8192u + (uint32_t)(j & 3) * 4u
                                               : (uint32_t)(j >> 6) * 8192u + (uint32_t)(j & 7) * 2u);
        const uint32_t och = sizeof(Tout) == 4 ? (uint32_t)((j & 31) >> 2) : (uint32_t)((j & 63) >> 3);
        bool ok;
        {
            float x[32];
            const float* s0 = (A.S0 && !tr) ? A.S0 + ((size_t)bh * kD + j) * kD + 32 * cg : nullptr;
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
                const float4 t = s0 ? *reinterpret_cast<const float4*>(s0 + e) : make_float4(0.f, 0.f, 0.f, 0.f);
                x[e] = t.x;
                x[e + 1] = t.y;
                x[e + 2] = t.z;
                x[e + 3] = t.w;
            }
            if (tr) {  // transition chain: the identity
#pragma unroll
                for (int e = 0; e < 32; ++e) x[e] = (j == 32 * cg + e) ? 1.f : 0.f;
            }
            hand_over(x);
            ok = decay(x, 0);
        }
        for (int c = 0; ok && c < NC; ++c) {
            const int sb = c & 1;
            const uint32_t tD1 = tbase + kTD1 + sb * 128;
            // ---- Delta^T[j][r] = U^T[j][r] - (S W^T)[j][r], r in [16 cg, 16 cg + 16), into TMEM
            if (!wait(&fullU[sb], (c >> 1) & 1) || !wait(&barA[sb], (c >> 1) & 1)) break;
            tc_fence_after();
            {
                float x[16], u[16];
                tmem_ld16(tD1 + lane_off + 16 * cg, x);
                if (tr) {  // transition chain: no write (v = 0 gives U = 0)
#pragma unroll
                    for (int e = 0; e < 16; ++e) u[e] = 0.f;
                } else {
                    unpack8h(ld16(sUT(sb) + kmajor_off(j, 16 * cg, 128)), u);
                    unpack8h(ld16(sUT(sb) + kmajor_off(j, 16 * cg + 8, 128)), u + 8);
                }
                tmem_ld_wait();
                uint32_t w[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) w[e] = pack2h(u[2 * e] - x[2 * e], u[2 * e + 1] - x[2 * e + 1]);
                tmem_st8(tbase + kTDelta + lane_off + 8 * cg, w);
                tmem_st_wait();  // also completes the D3 store of hand_over
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&deltaReady);
            // ---- S_{c+1} = gamma_C S_c + Delta^T K~ (D3): on to chunk c + 1, or out as S_T
            if (!wait(&barC, c & 1)) break;
            tc_fence_after();
            float x[32];
            tmem_ld32(tD3, x);
            tmem_ld_wait();
            if (c + 1 < NC) {
                hand_over(x);
            } else if ((tr ? A.S_T2 : A.S_T) != nullptr) {
                float* dst = (tr ? A.S_T2 : A.S_T) + ((size_t)bh * kD + j) * kD + 32 * cg;
#pragma unroll
                for (int e = 0; e < 32; e += 4)
                    *reinterpret_cast<float4*>(dst + e) = make_float4(x[e], x[e + 1], x[e + 2], x[e + 3]);
            }
            // ---- output of chunk c into the staging buffer sO(sb)
            if (!wait(&barB, c & 1) || !wait(&oFree[sb], (c >> 1) & 1)) break;
            tc_fence_after();
            {
                float x[16];
                tmem_ld16(tD1 + 64 + lane_off + 16 * cg, x);
                tmem_ld_wait();
                uint8_t* o = sO(sb) + ob;
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    uint8_t* p = o + e * 128 + ((och ^ (uint32_t)(e & 7)) << 4);
                    if (sizeof(Tout) == 4) *reinterpret_cast<float*>(p) = A.scale * x[e];
                    else *reinterpret_cast<__nv_bfloat16*>(p) = __float2bfloat16_rn(A.scale * x[e]);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&oStaged);
            // ---- gamma_C(c + 1) S_{c+1} into D3 while chunk c + 1's first product runs
            if (c + 1 < NC && !decay(x, c + 1)) break;
        }
    }
}

// Two-pass state kernel: one CTA per (b, h), hand-off blocks from the workspace. For the segment
// scan, CTAs n_data .. 2 n_data - 1 run the transition chains of the same heads (output map mo2).
template <typename Tout>
__global__ void __launch_bounds__(kStateThreads, 1)
chunk_state_kernel(const __grid_constant__ CUtensorMap mo, const __grid_constant__ CUtensorMap mo2, StateArgs A,
                   const uint8_t* __restrict__ ws) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag;
    const int warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) abort_flag = 0;
    if (warp == 0) {
        tmem_alloc(&tmem_base, kStateTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const bool tr = (int)blockIdx.x >= A.n_data;
    const int bh = tr ? (int)blockIdx.x - A.n_data : (int)blockIdx.x;
    const WorkspaceSource src{ws + (size_t)bh * A.NC * kHandoffStride, kHandoffStride};
    state_body<Tout>(tr ? &mo2 : &mo, A, bh, src, align1024(smem_raw), tmem_base, &abort_flag, tr);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem_base, kStateTmemCols);
}

// ------------------------------------------------------------------- fused kernel --
// Both passes in one cooperative launch: CTAs 0 .. BH-1 run the state pass of head bh = blockIdx.x,
// the other CTAs run two prep pipelines each (warps 0-7 and 8-15; warps 16-17 idle). The prep
// pipelines claim tasks from a counter in the order the state passes consume them (chunk index
// outermost: tau = c * BH + bh) and write each hand-off block into ring slot c % depth of
// its head, after the head's state pass has copied out chunk c - depth; a release flag per slot
// publishes the block. All CTAs are co-resident (cooperative launch), tasks are claimed in
// increasing order and the state passes consume in order, so the earliest unfinished task can
// always proceed. The ring stays in L2: the hand-off never makes a round trip to DRAM.
constexpr uint32_t kPrepPipeBytes = kPrepBytesScalar;  // one pipeline's shared memory (1024-aligned)
static_assert(kPrepPipeBytes % 1024 == 0, "pipeline shared memory must keep 1024-byte alignment");
static_assert(2 * (kPrepBytesScalar + 1024 + 1024 + 64) <= 233472, "two prep pipelines per SM");
constexpr uint32_t kFusedSmem = (2 * kPrepPipeBytes > kStateSmem - 1024 ? 2 * kPrepPipeBytes : kStateSmem - 1024) + 1024;
constexpr int kFusedMaxHeads = 100;  // B * H above this runs the two-pass path (too few SMs left for prep)
static_assert(kPrepBytesChannel <= kFusedSmem - 1024, "the channel gate's prep pipeline fits a fused CTA");

struct RingArgs {
    uint8_t* ring;     // [BH][depth] hand-off blocks
    int* ready;        // [BH][depth]
    int* consumed;     // [BH]
    int* next_task;    // prep tasks claimed so far (one counter, counted from task c1 * BH)
    const uint8_t* pre;  // [BH][c1] blocks of the chunks below c1, written by chunk_prep_kernel before
    int BH, c1;
    int depth;         // ring slots per head: kRing, or every chunk from c1 on when c1 > 0
};

template <int MODE, bool PRO, bool EW>
__device__ void prep_role(const CUtensorMap* mq, const CUtensorMap* mk, const CUtensorMap* mv, const PrepArgs& P,
                          const RingArgs& R, uint8_t* sm, uint32_t tbase, volatile int* abort) {
    __shared__ uint64_t pbars[2][4];
    __shared__ volatile int go[2];
    __shared__ volatile int claimed[2];
    // the channel gate's pipeline takes most of the shared memory: one per CTA (warps 0-7)
    constexpr int kPipes = MODE == GDR_DECAY_CHANNEL ? 1 : 2;
    const int tid = threadIdx.x, warp = tid >> 5;
    const int pipe = warp >> 3;  // pipelines 0 .. kPipes - 1; the other warps idle
    const int lt = tid & 255;
    if (tid == 0) {
        for (int i = 0; i < 2; ++i)
            for (int k = 0; k < 4; ++k) mbar_init(&pbars[i][k], 1);
        fence_mbar_init();
    }
    if (pipe < kPipes) prep_init<MODE>(PrepSmem{sm + pipe * kPrepPipeBytes, nullptr, 0, 0}, lt);
    __syncthreads();
    // a head's chain consumes a chunk about every 2 us and a pipeline prepares one in about 11 us:
    // 6 pipelines per head keep the rings full; more would only wait on ring slots
    if (pipe >= kPipes || (int)blockIdx.x - R.BH >= (6 / kPipes) * R.BH + 4) return;
    const PrepSmem ps{sm + pipe * kPrepPipeBytes, pbars[pipe], tbase + (uint32_t)pipe * kPrepTmemCols, 1 + 2 * pipe};
    const int n_tasks = P.NC * R.BH;
    uint32_t it = 0, n_copies = 0;  // tasks so far; channel-gate tile copies so far (mbarrier parities)
    for (;; ++it) {
        // claim the next task in consumption order (a pipeline claims only after finishing its
        // previous task, so claims, like the state passes' reads, go in increasing order). Claiming
        // one task ahead, to load its tile during the one before, was measured slower: the chains
        // wait longer for the earliest blocks.
        if (lt == 0) claimed[pipe] = R.c1 * R.BH + atomicAdd(R.next_task, 1);
        named_bar(ps.bar_id, kPrepThreads);
        const int tau = claimed[pipe];
        named_bar(ps.bar_id, kPrepThreads);  // every thread has read it before the next claim
        if (tau >= n_tasks) break;
        const int c = tau / R.BH, bh = tau % R.BH;
        const int slot = c % R.depth;
        if (lt == 0)
            go[pipe] = c - R.depth < R.c1 || flag_wait_geq(R.consumed + bh, c - R.depth + 1, P.status, abort, 2048);
        named_bar(ps.bar_id, kPrepThreads);
        if (!go[pipe]) break;
        uint8_t* out = R.ring + ((size_t)bh * R.depth + slot) * kHandoffStride;
        prep_chunk<MODE, PRO, EW>(P, mq, mk, mv, ps, bh / P.H, bh % P.H, c, out, it, lt, n_copies, 0, 0, -1, false);
        if (lt == 0) {  // every write of the block (generic stores before prep_chunk's last barrier, bulk stores)
            bulk_wait<0>();
            fence_proxy_async_global();
            __threadfence();
            st_release_gpu(R.ready + bh * R.depth + slot, c + 1);
        }
    }
}

template <int MODE, typename Tout, bool PRO, bool EW>
__global__ void __launch_bounds__(kStateThreads, 1)
chunk_fused_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
                   const __grid_constant__ CUtensorMap mv, const __grid_constant__ CUtensorMap mo, PrepArgs P,
                   StateArgs A, RingArgs R) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag;
    const int warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) abort_flag = 0;
    if (warp == 0) {
        tmem_alloc(&tmem_base, kStateTmemCols);  // 512: the state pass, or two prep pipelines x 256
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    uint8_t* sm = align1024(smem_raw);
    if ((int)blockIdx.x < R.BH) {
        const int bh = blockIdx.x;
        const RingSource src{R.pre + (size_t)bh * R.c1 * kHandoffStride,
                             R.ring + (size_t)bh * R.depth * kHandoffStride, R.ready + bh * R.depth, R.consumed + bh,
                             R.c1, R.depth};
        state_body<Tout>(&mo, A, bh, src, sm, tmem_base, &abort_flag);
    } else {
        prep_role<MODE, PRO, EW>(&mq, &mk, &mv, P, R, sm, tmem_base, &abort_flag);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem_base, kStateTmemCols);
}

// ---------------------------------------------------------------------- host --
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (fn == nullptr) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// 4-D map over a [B, T, H, 128] tensor: box of `box_cols` elements x 1 head x 64 tokens x 1 batch,
// 128-byte swizzle. Tokens past T read as zero and are not written.
cudaError_t make_map(CUtensorMap* map, const void* base, CUtensorMapDataType type, int esize, int B, int T, int H,
                     int box_cols) {
    EncodeTiledFn enc = encode_fn();
    if (enc == nullptr) return cudaErrorNotSupported;
    const cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)kD * esize, (cuuint64_t)H * kD * esize, (cuuint64_t)T * H * kD * esize};
    const cuuint32_t box[4] = {(cuuint32_t)box_cols, 1, (cuuint32_t)kC, 1};
    const cuuint32_t es[4] = {1, 1, 1, 1};
    const CUresult r = enc(map, type, 4, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                           CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int MODE, bool PRO, bool EW = false>
cudaError_t launch_prep(const ChunkProblem& p, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                        int NC, int NCp, uint8_t* blocks, cudaStream_t stream) {
    auto kern = chunk_prep_kernel<MODE, PRO, EW>;
    const uint32_t smem = (MODE == GDR_DECAY_CHANNEL ? kPrepBytesChannel : kPrepBytesScalar) + 1024;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    // the whole unified L1 / shared array as shared memory, so that two pipelines fit per SM
    err = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    if (err != cudaSuccess) return err;
    PrepArgs P{p.g, p.beta, p.T, p.H, NC, p.status, p.prologue, p.gate_scale, p.erase, p.write};
    int dev = 0, sms = 0;
    if ((err = cudaGetDevice(&dev)) != cudaSuccess) return err;
    if ((err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return err;
    // pipelines per SM: two for DeltaNet and the scalar gate (2 x (kPrepBytesScalar + 1,024 alignment
    // + 1,024 reserved + static) bytes fit in the SM's 228 KiB), one for the channel gate
    const int per_sm = MODE == GDR_DECAY_CHANNEL ? 1 : 2;
    const int n_tasks = NCp * p.H * p.B;
    const int grid = n_tasks < sms * per_sm ? n_tasks : sms * per_sm;
    kern<<<grid, kPrepThreads, smem, stream>>>(mq, mk, mv, P, blocks, NCp, n_tasks);
    profile_after_launch(stream);
    return cudaGetLastError();
}

template <typename Tout>
cudaError_t launch_state(const ChunkProblem& p, const CUtensorMap& mo, int NC, cudaStream_t stream) {
    auto kern = chunk_state_kernel<Tout>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kStateSmem);
    if (err != cudaSuccess) return err;
    StateArgs A{p.S0, p.S_T, p.T, p.H, NC, p.scale, p.status, p.B * p.H, nullptr};
    kern<<<p.B * p.H, kStateThreads, kStateSmem, stream>>>(mo, mo, A, static_cast<const uint8_t*>(p.workspace));
    profile_after_launch(stream);
    return cudaGetLastError();
}

// The fused kernel serves up to kFusedMaxHeads heads (the channel gate, and Gated DeltaNet-2 with it,
// with one prep pipeline per CTA: two do not fit in shared memory); larger B * H use two passes.
bool use_fused(int B, int H) { return (size_t)B * H <= kFusedMaxHeads; }

// Chunks per head the fused kernel takes pre-computed from a prep kernel that runs before it on
// all SMs. In the fused kernel the kSMs - BH prep CTAs must keep up with the BH chains: a chain
// takes chain_per_task(BH) times as long per chunk as a prep CTA (two pipelines) per task, so they
// produce the last NC - c1 chunks in time if (NC - c1) * BH <= NC * (kSMs - BH) * chain_per_task;
// the remaining chunks are prepared beforehand with every SM. (A fixed SM count keeps the result,
// and with it the workspace size, a host-only function of the shape.)
constexpr int kSMs = 148;
constexpr int kHybridMinHeads = 57;  // below, the fused kernel alone is faster (measured at 48 heads)
// Measured at T = 4096 (64 chunks), the best of 0.32 / 0.35 / 0.38 / 0.42: 0.35 at 64 heads (c1 = 35,
// 229.9 us; 0.38 within 1 us), 0.32 at 80 heads (c1 = 47, 265.6 vs 270.8 us at 0.35) and at 96
// heads (c1 = 53, 303.5 vs 311.6 us): the prep CTAs slow down as they get fewer and the chains
// more. Linear in between.
double chain_per_task(int BH) {
    const double t = (BH - 64) / 16.0;
    return 0.35 - 0.03 * (t < 0.0 ? 0.0 : t > 1.0 ? 1.0 : t);
}
// The channel gate: one prep pipeline per CTA, each task slower (more exponentials, and 112 registers
// in the fused kernel against 240 alone); the chain about 2 us per chunk. Measured at T = 8192, the
// best of 0.13 / 0.16 / 0.19 / 0.22 at 32, 64 and 96 heads: 0.13 (64 heads: c1 = 107 of 128, 813 us,
// against 835 at 0.16 and 902 for two passes; the fused kernel then at about the chain's own time).
constexpr double kChainPerTaskChannel = 0.13;
// Gated DeltaNet-2 (ew): the channel gate's prep with the erase / write gates, about 1.6 times as long
// per task. Measured at the KDA workload's shape (64 heads, 128 chunks): 0.08 (c1 = 115) 1193 us,
// against 1224 us at 0.06, 1227 us at 0.10 and 1291 us for two passes.
constexpr double kChainPerTaskGdn2 = 0.08;
// With the mixer prologue (pro) each prep task does more, so where chunks are pre-computed at all,
// more of them are (the ratio scaled by kProChainScale). A larger c1 keeps the call inside the plain
// call's workspace: pre-computed and ring blocks total one per chunk either way, and the flags shrink.
constexpr double kProChainScale = 0.75;
int precomputed_for(double k, int BH, int NC) {
    const double f = 1.0 - k * (kSMs - BH) / (double)BH;
    if (f <= 0.0) return 0;
    const int c1 = (int)(f * NC + 0.999);
    return c1 < NC ? c1 : NC;
}
int fused_precomputed_chunks(int BH, int NC, int mode, bool ew = false, bool pro = false) {
    const bool ch = mode == GDR_DECAY_CHANNEL;
    if (!ch && BH < kHybridMinHeads) return 0;
    const double k = ch ? (ew ? kChainPerTaskGdn2 : kChainPerTaskChannel) : chain_per_task(BH);
    const int c1 = precomputed_for(k, BH, NC);
    if (c1 == 0 || !pro) return c1;
    const int c1p = precomputed_for(k * kProChainScale, BH, NC);
    return c1p > c1 ? c1p : c1;
}
size_t pre_bytes(int BH, int NC, int mode, bool ew, bool pro = false) {
    return (size_t)BH * fused_precomputed_chunks(BH, NC, mode, ew, pro) * kHandoffStride;
}
// Ring slots per head. With chunks pre-computed, the chains spend their first c1 chunks on those
// while the fused kernel's prep CTAs run ahead: a slot for every later chunk keeps them from
// stalling on a full ring in that time (the blocks then mostly live in DRAM, not L2).
int ring_depth(int BH, int NC, int mode, bool ew, bool pro = false) {
    const int c1 = fused_precomputed_chunks(BH, NC, mode, ew, pro);
    return c1 > 0 ? NC - c1 : kRing;
}
size_t ring_bytes(int BH, int NC, int mode, bool ew, bool pro = false) {
    return (size_t)BH * ring_depth(BH, NC, mode, ew, pro) * kHandoffStride;
}
size_t flag_bytes(int BH, int NC, int mode, bool ew, bool pro = false) {
    return ((size_t)(BH * (ring_depth(BH, NC, mode, ew, pro) + 1) + 1) * sizeof(int) + 255) & ~size_t(255);
}

template <int MODE, typename Tout, bool PRO, bool EW = false>
cudaError_t launch_fused(const ChunkProblem& p, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                         const CUtensorMap& mo, int NC, cudaStream_t stream) {
    auto kern = chunk_fused_kernel<MODE, Tout, PRO, EW>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kFusedSmem);
    if (err != cudaSuccess) return err;
    int dev = 0, sms = 0, coop = 0, per_sm = 0;
    if ((err = cudaGetDevice(&dev)) != cudaSuccess) return err;
    if ((err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return err;
    if ((err = cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev)) != cudaSuccess) return err;
    if ((err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kStateThreads, kFusedSmem)) != cudaSuccess)
        return err;
    const int BH = p.B * p.H;
    const int grid = sms * per_sm;
    if (!coop || per_sm < 1 || grid - BH < 8) return cudaErrorCooperativeLaunchTooLarge;
    // workspace: [pre-computed blocks, BH x c1][ring, BH x depth][flags]
    uint8_t* ws = static_cast<uint8_t*>(p.workspace);
    const int c1 = fused_precomputed_chunks(BH, NC, MODE, EW, PRO), depth = ring_depth(BH, NC, MODE, EW, PRO);
    uint8_t* ring = ws + pre_bytes(BH, NC, MODE, EW, PRO);
    int* flags = reinterpret_cast<int*>(ring + ring_bytes(BH, NC, MODE, EW, PRO));
    RingArgs R{ring, flags, flags + (size_t)BH * depth, flags + (size_t)BH * (depth + 1), ws, BH, c1, depth};
    if ((err = cudaMemsetAsync(flags, 0, flag_bytes(BH, NC, MODE, EW, PRO), stream)) != cudaSuccess) return err;
    if (c1 > 0 && (err = launch_prep<MODE, PRO, EW>(p, mq, mk, mv, NC, c1, ws, stream)) != cudaSuccess) return err;
    PrepArgs P{p.g, p.beta, p.T, p.H, NC, p.status, p.prologue, p.gate_scale, p.erase, p.write};
    StateArgs A{p.S0, p.S_T, p.T, p.H, NC, p.scale, p.status, p.B * p.H, nullptr};
    CUtensorMap aq = mq, ak = mk, av = mv, ao = mo;
    void* args[] = {&aq, &ak, &av, &ao, &P, &A, &R};
    err = cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(kern), dim3(grid), dim3(kStateThreads), args,
                                      kFusedSmem, stream);
    profile_after_launch(stream);
    return err;
}

template <bool PRO>
cudaError_t launch_fused_mode(const ChunkProblem& p, const CUtensorMap& mq, const CUtensorMap& mk,
                              const CUtensorMap& mv, const CUtensorMap& mo, int NC, cudaStream_t stream) {
    const bool bf = p.o_dtype == GDR_BF16;
    if (p.mode == GDR_DECAY_NONE)
        return bf ? launch_fused<GDR_DECAY_NONE, __nv_bfloat16, PRO>(p, mq, mk, mv, mo, NC, stream)
                  : launch_fused<GDR_DECAY_NONE, float, PRO>(p, mq, mk, mv, mo, NC, stream);
    if (p.mode == GDR_DECAY_CHANNEL)
        return bf ? launch_fused<GDR_DECAY_CHANNEL, __nv_bfloat16, PRO>(p, mq, mk, mv, mo, NC, stream)
                  : launch_fused<GDR_DECAY_CHANNEL, float, PRO>(p, mq, mk, mv, mo, NC, stream);
    return bf ? launch_fused<GDR_DECAY_SCALAR, __nv_bfloat16, PRO>(p, mq, mk, mv, mo, NC, stream)
              : launch_fused<GDR_DECAY_SCALAR, float, PRO>(p, mq, mk, mv, mo, NC, stream);
}

template <bool PRO>
cudaError_t launch_prep_mode(const ChunkProblem& p, const CUtensorMap& mq, const CUtensorMap& mk,
                             const CUtensorMap& mv, int NC, uint8_t* ws, cudaStream_t stream) {
    switch (p.mode) {
        case GDR_DECAY_NONE: return launch_prep<GDR_DECAY_NONE, PRO>(p, mq, mk, mv, NC, NC, ws, stream);
        case GDR_DECAY_SCALAR: return launch_prep<GDR_DECAY_SCALAR, PRO>(p, mq, mk, mv, NC, NC, ws, stream);
        case GDR_DECAY_CHANNEL: return launch_prep<GDR_DECAY_CHANNEL, PRO>(p, mq, mk, mv, NC, NC, ws, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

bool chunk_tc_supported(int dk, int dv, int chunk, int dtype, int o_dtype) {
    return dtype == GDR_BF16 && (o_dtype == GDR_F32 || o_dtype == GDR_BF16) && dk == kD && dv == kD && chunk == kC;
}

size_t chunk_tc_workspace_bytes(int B, int T, int H, int, int, int, int mode, bool ew) {
    const int NC = (T + kC - 1) / kC, BH = B * H;
    if (use_fused(B, H))
        return pre_bytes(BH, NC, mode, ew) + ring_bytes(BH, NC, mode, ew) + flag_bytes(BH, NC, mode, ew);
    return (size_t)BH * NC * kHandoffStride;
}

int chunk_tc_plan(int B, int T, int H, int, int, int, int mode, int* precomputed_chunks) {
    const int NC = (T + kC - 1) / kC;
    const int c1 = use_fused(B, H) ? fused_precomputed_chunks(B * H, NC, mode) : 0;
    if (precomputed_chunks != nullptr) *precomputed_chunks = c1;
    if (!use_fused(B, H)) return GDR_PLAN_TWO_PASS;
    return c1 > 0 ? GDR_PLAN_PREP_FUSED : GDR_PLAN_FUSED;
}

int chunk_tc_launches(int B, int T, int H, int, int, int, int mode) {
    if (!use_fused(B, H)) return 2;
    return fused_precomputed_chunks(B * H, (T + kC - 1) / kC, mode) > 0 ? 2 : 1;
}

cudaError_t launch_chunk_tc(const ChunkProblem& p, cudaStream_t stream) {
    const int NC = (p.T + kC - 1) / kC;
    CUtensorMap mq, mk, mv, mo;
    cudaError_t err;
    if ((err = make_map(&mq, p.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.B, p.T, p.H, 64)) != cudaSuccess) return err;
    if ((err = make_map(&mk, p.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.B, p.T, p.H, 64)) != cudaSuccess) return err;
    if ((err = make_map(&mv, p.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.B, p.T, p.H, 64)) != cudaSuccess) return err;
    if (p.o_dtype == GDR_BF16)
        err = make_map(&mo, p.o, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.B, p.T, p.H, 64);
    else
        err = make_map(&mo, p.o, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, p.B, p.T, p.H, 32);
    if (err != cudaSuccess) return err;
    // Gated DeltaNet-2: the channel gate's prep with the erase / write gates
    const bool ew = p.erase != nullptr;
    if (ew && (p.mode != GDR_DECAY_CHANNEL || p.prologue)) return cudaErrorInvalidValue;
    if (use_fused(p.B, p.H)) {
        if (ew)
            return p.o_dtype == GDR_BF16
                       ? launch_fused<GDR_DECAY_CHANNEL, __nv_bfloat16, false, true>(p, mq, mk, mv, mo, NC, stream)
                       : launch_fused<GDR_DECAY_CHANNEL, float, false, true>(p, mq, mk, mv, mo, NC, stream);
        return p.prologue ? launch_fused_mode<true>(p, mq, mk, mv, mo, NC, stream)
                          : launch_fused_mode<false>(p, mq, mk, mv, mo, NC, stream);
    }
    uint8_t* ws = static_cast<uint8_t*>(p.workspace);
    if (ew) {
        err = launch_prep<GDR_DECAY_CHANNEL, false, true>(p, mq, mk, mv, NC, NC, ws, stream);
    } else {
        err = p.prologue ? launch_prep_mode<true>(p, mq, mk, mv, NC, ws, stream)
                         : launch_prep_mode<false>(p, mq, mk, mv, NC, ws, stream);
    }
    if (err != cudaSuccess) return err;
    if (p.o_dtype == GDR_BF16) return launch_state<__nv_bfloat16>(p, mo, NC, stream);
    return launch_state<float>(p, mo, NC, stream);
}

size_t chunk_tc_pair_workspace_bytes(int B, int T, int H) {
    return (size_t)B * H * ((T + kC - 1) / kC) * kHandoffStride;
}

// Segment scan: the prep pass over every chunk, then one state-kernel launch whose first B * H CTAs
// run the data chains (o -> p.o, S_T -> p.S_T) and whose other B * H CTAs run the transition chains
// over the same hand-off blocks (identity state, no write: per-token read-outs -> o2, S_T -> S_T2).
// p.o and o2 are fp32.
cudaError_t launch_chunk_tc_pair(const ChunkProblem& p, void* o2, float* S_T2, cudaStream_t stream) {
    const int NC = (p.T + kC - 1) / kC;
    CUtensorMap mq, mk, mv, mo, mo2;
    cudaError_t err;
    if ((err = make_map(&mq, p.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.B, p.T, p.H, 64)) != cudaSuccess) return err;
    if ((err = make_map(&mk, p.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.B, p.T, p.H, 64)) != cudaSuccess) return err;
    if ((err = make_map(&mv, p.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.B, p.T, p.H, 64)) != cudaSuccess) return err;
    if ((err = make_map(&mo, p.o, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, p.B, p.T, p.H, 32)) != cudaSuccess) return err;
    if ((err = make_map(&mo2, o2, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, p.B, p.T, p.H, 32)) != cudaSuccess) return err;
    uint8_t* ws = static_cast<uint8_t*>(p.workspace);
    err = p.prologue ? launch_prep_mode<true>(p, mq, mk, mv, NC, ws, stream)
                     : launch_prep_mode<false>(p, mq, mk, mv, NC, ws, stream);
    if (err != cudaSuccess) return err;
    auto kern = chunk_state_kernel<float>;
    if ((err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kStateSmem)) != cudaSuccess)
        return err;
    const int BH = p.B * p.H;
    StateArgs A{p.S0, p.S_T, p.T, p.H, NC, p.scale, p.status, BH, S_T2};
    kern<<<2 * BH, kStateThreads, kStateSmem, stream>>>(mo, mo2, A, ws);
    profile_after_launch(stream);
    return cudaGetLastError();
}

}  // namespace gdr
