// gdr_chunk_tc.cu -- chunked gated delta-rule forward on the 5th-generation tensor cores.
//
// bf16 q/k/v, d_k = d_v = 128, chunk C = 64; fp16 MMA operands, fp32 accumulation (TMEM) and fp32
// state (registers).
// The chunk form ("linear attention and its gated descendants", Chunkwise Parallel Form, with the
// WY/UT compact form of a chunk of delta-rule updates from "Linear Attention & DeltaNet", item 3),
// with Gamma the inclusive cumulative log-decay inside the chunk and gamma = exp(Gamma):
//
//   A  = strictly_lower(diag(beta) (K*gamma)(K/gamma)^T),  T = (I + A)^-1      (UT transform)
//   W  = T diag(beta) (K*gamma),  U = T diag(beta) V                           (WY factors)
//   P  = causal_incl_diag((Q*gamma)(K/gamma)^T)
//   Delta = U - W S^T
//   O  = scale [ (Q*gamma) S^T + P Delta ]
//   S <- S Diag(gamma_C) + Delta^T (K * gamma_C / gamma)
//
// Two kernels. The prep kernel runs one CTA per chunk, all chunks in parallel: it computes the
// S-independent factors (two tcgen05 GEMM groups around a CUDA-core triangular solve) and writes
// them to the workspace as ready-to-use, 128-byte-swizzled shared-memory operand images. The state
// kernel runs one CTA per (b, h) and walks the chunks in order: it bulk-copies each chunk's images
// into a double-buffered stage and runs the three S-dependent tcgen05 GEMM groups; the fp32 state
// lives in registers and enters the MMAs as an fp16 copy in shared memory.
//
// Decay handling: for the scalar gate the Gram products use raw K, Q and are scaled elementwise by
// exp(Gamma_r - Gamma_i) <= 1 afterwards (safe for any g <= 0). For the channel gate the factors
// are folded into the operands around a mid-chunk reference Gamma_ref:
// (K e^{Gamma - Gamma_ref})(K e^{Gamma_ref - Gamma})^T. A factor above the fp16 range (a
// within-chunk spread of the cumulative log-decay beyond about 22 on one channel) is detected and
// reported as GDR_ERR_RANGE through the status word.
#include <cuda_fp16.h>

#include "gdr_sm100.cuh"

namespace gdr {
namespace {

using namespace sm100;

constexpr int kC = 64;    // chunk length
constexpr int kD = 128;   // d_k = d_v

// Per-chunk hand-off block in the workspace (byte offsets). Every image is laid out exactly as
// the state kernel's MMAs read it from shared memory.
constexpr uint32_t kOffWT = 0;            // W^T:          MN-major, K = d_k (128 rows) x N = C (64)
constexpr uint32_t kOffQG = 16384;        // Q*gamma:      K-major,  N = C (64 rows)  x K = d_k (128)
constexpr uint32_t kOffKT = 32768;        // K*gamma_C/gamma: MN-major, K = C (64 rows) x N = d_k (128)
constexpr uint32_t kOffUT = 49152;        // U^T:          plain row-major fp16 [d_v][C]
constexpr uint32_t kOffP = 65536;         // P:            K-major,  N = C (r, 64 rows) x K = C (i, 64)
constexpr uint32_t kOffGam = 73728;       // gamma_C:      128 fp32 (per key channel)
constexpr uint32_t kHandoffBytes = 74240;   // bytes copied per chunk (multiple of 16)
constexpr uint32_t kHandoffStride = 74752;  // per-chunk stride (multiple of 1024)

constexpr int kPrepThreads = 128;
constexpr int kStateThreads = 256;

// prep kernel shared memory (offsets from a 1024-aligned base)
constexpr uint32_t kPrepAG = 0;           // [K'; Q'] K-major 128 rows x 128      32 KiB
constexpr uint32_t kPrepBG = 32768;       // K'' K-major 64 rows x 128            16 KiB
constexpr uint32_t kPrepKG = 49152;       // K*gamma K-major 64 x 128             16 KiB
constexpr uint32_t kPrepV = 65536;        // V K-major 64 x 128                   16 KiB
constexpr uint32_t kPrepTB = 81920;       // T diag(beta) K-major 64 x 64          8 KiB
constexpr uint32_t kPrepGam = 90112;      // Gamma fp32 [64][128] (channel) or [64] 32 KiB
constexpr uint32_t kPrepBeta = 122880;    // beta fp32 [64]
constexpr uint32_t kPrepSmem = 123136 + 1024;
// solve scratch, aliasing the Gram operands once the Gram MMA has completed
constexpr uint32_t kPrepA = 0;            // A fp32 [64][65]
constexpr uint32_t kPrepT = 17408;        // T fp32 [64][65]
constexpr uint32_t kPrepX = 34816;        // block products fp32 [3][16][17]
constexpr int kLd = 65;

// state kernel shared memory
constexpr uint32_t kStS = 2 * kHandoffStride;    // S fp16 K-major 128 x 128   32 KiB
constexpr uint32_t kStDT = kStS + 32768;         // Delta^T fp16 K-major 128 x 64 16 KiB
constexpr uint32_t kStateSmem = kStDT + 16384 + 1024;

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// MMA operands are fp16 (10-bit mantissa): bf16 inputs convert to it exactly, and with bf16
// operands the rounding of the intermediate factors alone exceeded the 2e-2 * rms(o) parity bar.
__device__ __forceinline__ uint32_t pack2(float a, float b) {
    __half2 t = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&t);
}

__device__ __forceinline__ uint4 pack8(const float* f) {
    return make_uint4(pack2(f[0], f[1]), pack2(f[2], f[3]), pack2(f[4], f[5]), pack2(f[6], f[7]));
}

// 8 bf16 (inputs) to fp32
__device__ __forceinline__ void unpack8(uint4 u, float* f) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __nv_bfloat162 t = *reinterpret_cast<const __nv_bfloat162*>(&w[i]);
        f[2 * i] = __low2float(t);
        f[2 * i + 1] = __high2float(t);
    }
}

// 8 fp16 (operand images) to fp32
__device__ __forceinline__ void unpack8h(uint4 u, float* f) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __half2 t = *reinterpret_cast<const __half2*>(&w[i]);
        f[2 * i] = __low2float(t);
        f[2 * i + 1] = __high2float(t);
    }
}

constexpr float kF16Max = 65504.f;

__device__ __forceinline__ void st16(void* p, uint4 v) { *reinterpret_cast<uint4*>(p) = v; }

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// T = (I + A)^-1 for a 64 x 64 strictly-lower A (fp32, stride kLd). Diagonal 16 x 16 blocks by
// forward substitution, then block rows top-down: T_IJ = -T_II sum_{J<=K<I} A_IK T_KJ.
__device__ void unit_lower_inverse64(const float* __restrict__ A, float* __restrict__ Tm, float* __restrict__ X,
                                     int tid) {
    if (tid < 64) {
        const int base = (tid >> 4) * 16, j = tid & 15;
        float t[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            float acc = (r == j) ? 1.f : 0.f;
#pragma unroll
            for (int i = 0; i < r; ++i) acc = fmaf(-A[(base + r) * kLd + base + i], t[i], acc);
            t[r] = (r < j) ? 0.f : acc;
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) Tm[(base + r) * kLd + base + j] = t[r];
    } else {
        // zero the strictly-upper 16 x 16 blocks (6 blocks)
        for (int e = tid - 64; e < 6 * 256; e += 64) {
            const int blk = e >> 8, rr = (e >> 4) & 15, cc = e & 15;
            const int I = (blk < 3) ? 0 : (blk < 5 ? 1 : 2);
            const int J = (blk < 3) ? blk + 1 : (blk < 5 ? blk - 1 : 3);
            Tm[(16 * I + rr) * kLd + 16 * J + cc] = 0.f;
        }
    }
    __syncthreads();
    for (int I = 1; I < 4; ++I) {
        for (int e = tid; e < I * 256; e += kPrepThreads) {
            const int J = e >> 8, rr = (e >> 4) & 15, cc = e & 15;
            float acc = 0.f;
            for (int K = J; K < I; ++K)
#pragma unroll
                for (int m = 0; m < 16; ++m)
                    acc = fmaf(A[(16 * I + rr) * kLd + 16 * K + m], Tm[(16 * K + m) * kLd + 16 * J + cc], acc);
            X[J * 272 + rr * 17 + cc] = acc;
        }
        __syncthreads();
        for (int e = tid; e < I * 256; e += kPrepThreads) {
            const int J = e >> 8, rr = (e >> 4) & 15, cc = e & 15;
            float acc = 0.f;
            for (int m = 0; m <= rr; ++m) acc = fmaf(Tm[(16 * I + rr) * kLd + 16 * I + m], X[J * 272 + m * 17 + cc], acc);
            Tm[(16 * I + rr) * kLd + 16 * J + cc] = -acc;
        }
        __syncthreads();
    }
}

// ------------------------------------------------------------------------ prep --
template <int MODE>
__global__ void __launch_bounds__(kPrepThreads)
chunk_prep_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                  const __nv_bfloat16* __restrict__ v, const float* __restrict__ g, const float* __restrict__ beta,
                  int T, int H, int NC, uint8_t* __restrict__ ws, int* status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = align1024(smem_raw);
    uint8_t* sAG = sm + kPrepAG;
    uint8_t* sBG = sm + kPrepBG;
    uint8_t* sKG = sm + kPrepKG;
    uint8_t* sV = sm + kPrepV;
    uint8_t* sTB = sm + kPrepTB;
    float* sGam = reinterpret_cast<float*>(sm + kPrepGam);
    float* sBeta = reinterpret_cast<float*>(sm + kPrepBeta);
    __shared__ uint64_t bar;
    __shared__ uint32_t tmem_base;

    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int c0 = c * kC;
    const int n = min(kC, T - c0);
    const size_t tok0 = ((size_t)b * T + c0) * H + h;  // row r of the chunk is token tok0 + r * H
    uint8_t* out = ws + ((size_t)(b * H + h) * NC + c) * kHandoffStride;

    if (tid == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&tmem_base, 256);
        tmem_relinquish();
    }

    // ---- beta and the inclusive cumulative log-decay (rows past the tail repeat Gamma_{n-1})
    if (tid < kC) sBeta[tid] = (tid < n) ? beta[tok0 + (size_t)tid * H] : 0.f;
    if (MODE == GDR_DECAY_SCALAR) {
        if (warp == 0) {
            float x0 = (lane < n) ? g[tok0 + (size_t)lane * H] : 0.f;
            float x1 = (lane + 32 < n) ? g[tok0 + (size_t)(lane + 32) * H] : 0.f;
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
        }
    } else if (MODE == GDR_DECAY_CHANNEL) {
        float acc = 0.f;
        for (int r = 0; r < kC; ++r) {
            if (r < n) acc += g[(tok0 + (size_t)r * H) * kD + tid];
            sGam[r * kD + tid] = acc;
        }
    }
    __syncthreads();

    // ---- stage K, Q, V and the decay-scaled operands; write Q*gamma and K*gamma_C/gamma out
    const int ref = (n - 1) >> 1;  // channel mode: mid-chunk reference row
    bool range_bad = false;
    for (int it = 0; it < 8; ++it) {
        const int task = tid + kPrepThreads * it;
        const int r = task >> 4, col0 = (task & 15) * 8;
        float kx[8], qx[8], vx[8];
        if (r < n) {
            const size_t off = (tok0 + (size_t)r * H) * kD + col0;
            unpack8(*reinterpret_cast<const uint4*>(k + off), kx);
            unpack8(*reinterpret_cast<const uint4*>(q + off), qx);
            unpack8(*reinterpret_cast<const uint4*>(v + off), vx);
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) kx[e] = qx[e] = vx[e] = 0.f;
        }
        float ka[8], qa[8], kb[8], kg[8], qg[8], kt[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            if (MODE == GDR_DECAY_NONE) {
                ka[e] = kb[e] = kg[e] = kt[e] = kx[e];
                qa[e] = qg[e] = qx[e];
            } else if (MODE == GDR_DECAY_SCALAR) {
                const float G = sGam[r];
                const float gr = expf(G), tail = expf(sGam[kC - 1] - G);
                ka[e] = kb[e] = kx[e];
                qa[e] = qx[e];
                kg[e] = kx[e] * gr;
                qg[e] = qx[e] * gr;
                kt[e] = kx[e] * tail;
            } else {
                const float G = sGam[r * kD + col0 + e];
                const float Gr = sGam[ref * kD + col0 + e];
                const float GC = sGam[(kC - 1) * kD + col0 + e];
                const float up = expf(G - Gr), dn = expf(Gr - G), gr = expf(G);
                ka[e] = kx[e] * up;
                qa[e] = qx[e] * up;
                kb[e] = kx[e] * dn;
                if (!(up < kF16Max && dn < kF16Max)) range_bad = true;
                kg[e] = kx[e] * gr;
                qg[e] = qx[e] * gr;
                kt[e] = kx[e] * expf(GC - G);
            }
        }
        st16(sAG + kmajor_off(r, col0, 128), pack8(ka));
        st16(sAG + kmajor_off(kC + r, col0, 128), pack8(qa));
        st16(sBG + kmajor_off(r, col0, 64), pack8(kb));
        st16(sKG + kmajor_off(r, col0, 64), pack8(kg));
        st16(sV + kmajor_off(r, col0, 64), pack8(vx));
        st16(out + kOffQG + kmajor_off(r, col0, 64), pack8(qg));
        st16(out + kOffKT + mnmajor_off(r, col0, 64), pack8(kt));
    }
    if (MODE == GDR_DECAY_CHANNEL && range_bad) report_status(status, GDR_ERR_RANGE);
    {
        float gc = 1.f;
        if (MODE == GDR_DECAY_SCALAR) gc = expf(sGam[kC - 1]);
        if (MODE == GDR_DECAY_CHANNEL) gc = expf(sGam[(kC - 1) * kD + tid]);
        reinterpret_cast<float*>(out + kOffGam)[tid] = gc;
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // ---- Gram products: rows 0-63 K' K''^T, rows 64-127 Q' K''^T (M = 128, N = 64, K = 128)
    const uint32_t tG = tmem_base, tW = tmem_base + 64, tU = tmem_base + 128;
    if (tid == 0) {
        const uint32_t id = idesc_f16(128, 64, false, false);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
            mma_f16(tG, sdesc(smem_u32(sAG) + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024),
                     sdesc(smem_u32(sBG) + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024), id, ks > 0);
        mma_commit(&bar);
    }
    __syncwarp();
    mbar_wait(&bar, 0, status);
    tc_fence_after();

    float* sA = reinterpret_cast<float*>(sm + kPrepA);
    float* sT = reinterpret_cast<float*>(sm + kPrepT);
    float* sX = reinterpret_cast<float*>(sm + kPrepX);
    {
        const int rr = (warp & 1) * 32 + lane;  // chunk row of this thread's TMEM lane
        const uint32_t lane_addr = tG + ((uint32_t)(warp * 32) << 16);
        const float br = sBeta[rr];
        float Gr = 0.f;
        if (MODE == GDR_DECAY_SCALAR) Gr = sGam[rr];
        for (int half = 0; half < 2; ++half) {
            float x[32];
            tmem_ld32(lane_addr + half * 32, x);
            tmem_ld_wait();
            float p[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const int i = half * 32 + e;
                float d = 1.f;
                if (MODE == GDR_DECAY_SCALAR) d = (i <= rr) ? expf(Gr - sGam[i]) : 0.f;
                if (warp < 2) {
                    sA[rr * kLd + i] = (i < rr && rr < n) ? br * x[e] * d : 0.f;
                } else {
                    p[e] = (i <= rr && rr < n) ? x[e] * d : 0.f;
                }
            }
            if (warp >= 2) {
#pragma unroll
                for (int ci = 0; ci < 4; ++ci) st16(out + kOffP + kmajor_off(rr, half * 32 + ci * 8, 64), pack8(p + ci * 8));
            }
        }
    }
    tc_fence_before();
    __syncthreads();

    // ---- UT transform: T = (I + A)^-1, then T diag(beta) as the K-major B operand
    unit_lower_inverse64(sA, sT, sX, tid);
    for (int task = tid; task < 64 * 8; task += kPrepThreads) {
        const int r = task >> 3, i0 = (task & 7) * 8;
        float t8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) t8[e] = sT[r * kLd + i0 + e] * sBeta[i0 + e];
        st16(sTB + kmajor_off(r, i0, 64), pack8(t8));
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // ---- W^T = (K*gamma)^T (T diag beta)^T and U^T = V^T (T diag beta)^T (M = 128, N = 64, K = 64)
    if (tid == 0) {
        const uint32_t id = idesc_f16(128, 64, true, false);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            const uint64_t bd = sdesc(smem_u32(sTB) + ks * 32, 16, 1024);
            mma_f16(tW, sdesc(smem_u32(sKG) + ks * 2048, 8192, 1024), bd, id, ks > 0);
            mma_f16(tU, sdesc(smem_u32(sV) + ks * 2048, 8192, 1024), bd, id, ks > 0);
        }
        mma_commit(&bar);
    }
    __syncwarp();
    mbar_wait(&bar, 1, status);
    tc_fence_after();
    {
        const int row = warp * 32 + lane;  // d_k index for W^T, d_v index for U^T
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        for (int half = 0; half < 2; ++half) {
            float x[32];
            tmem_ld32(tW + lane_off + half * 32, x);
            tmem_ld_wait();
#pragma unroll
            for (int ci = 0; ci < 4; ++ci)
                st16(out + kOffWT + mnmajor_off(row, half * 32 + ci * 8, 128), pack8(x + ci * 8));
            tmem_ld32(tU + lane_off + half * 32, x);
            tmem_ld_wait();
#pragma unroll
            for (int ci = 0; ci < 4; ++ci) st16(out + kOffUT + row * 128 + (half * 32 + ci * 8) * 2, pack8(x + ci * 8));
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem_base, 256);
}

// ----------------------------------------------------------------------- state --
template <typename Tout>
__global__ void __launch_bounds__(kStateThreads, 1)
chunk_state_kernel(const uint8_t* __restrict__ ws, const float* S0, Tout* __restrict__ o, float* S_T, int T, int H,
                   int NC, float scale, int* status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = align1024(smem_raw);
    uint8_t* stage0 = sm;
    uint8_t* stage1 = sm + kHandoffStride;
    uint8_t* sS = sm + kStS;
    uint8_t* sDT = sm + kStDT;
    __shared__ uint64_t full[2], barA, barB;
    __shared__ uint32_t tmem_base;

    const int bh = blockIdx.x;
    const int b = bh / H, h = bh % H;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, half = warp >> 2;
    const int j = quad * 32 + lane;  // state row (d_v index) = TMEM lane
    const uint8_t* src = ws + (size_t)bh * NC * kHandoffStride;

    if (tid == 0) {
        mbar_init(&full[0], 1);
        mbar_init(&full[1], 1);
        mbar_init(&barA, 1);
        mbar_init(&barB, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&tmem_base, 256);
        tmem_relinquish();
    }

    // initial state: this thread holds S[j][64*half .. 64*half + 63] in fp32
    float s[64];
    {
        const float* s0 = S0 ? S0 + ((size_t)bh * kD + j) * kD + 64 * half : nullptr;
#pragma unroll
        for (int e = 0; e < 64; e += 4) {
            float4 t = s0 ? *reinterpret_cast<const float4*>(s0 + e) : make_float4(0.f, 0.f, 0.f, 0.f);
            s[e] = t.x;
            s[e + 1] = t.y;
            s[e + 2] = t.z;
            s[e + 3] = t.w;
        }
#pragma unroll
        for (int ci = 0; ci < 8; ++ci) st16(sS + kmajor_off(j, 64 * half + ci * 8, 128), pack8(s + ci * 8));
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {
        for (int st = 0; st < 2 && st < NC; ++st) {
            mbar_arrive_expect_tx(&full[st], kHandoffBytes);
            bulk_g2s(st ? stage1 : stage0, src + (size_t)st * kHandoffStride, kHandoffBytes, &full[st]);
        }
    }
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t tD1 = tmem_base, tD3 = tmem_base + 128;
    const int dv = kD;

    for (int c = 0; c < NC; ++c) {
        const int st = c & 1;
        uint8_t* S_ = st ? stage1 : stage0;
        mbar_wait(&full[st], (c >> 1) & 1, status);
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        // D1[:, 0:64] = S W^T ; D1[:, 64:128] = S (Q*gamma)^T   (M = 128, N = 64, K = 128)
        if (tid == 0) {
            const uint32_t idW = idesc_f16(128, 64, false, true);
            const uint32_t idQ = idesc_f16(128, 64, false, false);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint64_t ad = sdesc(smem_u32(sS) + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
                mma_f16(tD1, ad, sdesc(smem_u32(S_ + kOffWT) + ks * 2048, 16384, 1024), idW, ks > 0);
                mma_f16(tD1 + 64, ad, sdesc(smem_u32(S_ + kOffQG) + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024),
                         idQ, ks > 0);
            }
            mma_commit(&barA);
        }
        __syncwarp();
        mbar_wait(&barA, c & 1, status);
        tc_fence_after();
        // Delta^T[j][r] = U^T[j][r] - (S W^T)[j][r] for r in [32*half, 32*half + 32)
        {
            float x[32], u[32];
            tmem_ld32(tD1 + lane_off + 32 * half, x);
            const uint8_t* ut = S_ + kOffUT + j * 128 + 64 * half;
#pragma unroll
            for (int ci = 0; ci < 4; ++ci) unpack8h(*reinterpret_cast<const uint4*>(ut + ci * 16), u + ci * 8);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) u[e] -= x[e];
#pragma unroll
            for (int ci = 0; ci < 4; ++ci) st16(sDT + kmajor_off(j, 32 * half + ci * 8, 128), pack8(u + ci * 8));
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        // D1[:, 64:128] += Delta^T P^T (M = 128, N = 64, K = 64); D3 = Delta^T K~ (M = 128, N = 128, K = 64)
        if (tid == 0) {
            const uint32_t idP = idesc_f16(128, 64, false, false);
            const uint32_t idK = idesc_f16(128, 128, false, true);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const uint64_t ad = sdesc(smem_u32(sDT) + ks * 32, 16, 1024);
                mma_f16(tD1 + 64, ad, sdesc(smem_u32(S_ + kOffP) + ks * 32, 16, 1024), idP, true);
                mma_f16(tD3, ad, sdesc(smem_u32(S_ + kOffKT) + ks * 2048, 8192, 1024), idK, ks > 0);
            }
            mma_commit(&barB);
        }
        __syncwarp();
        mbar_wait(&barB, c & 1, status);
        tc_fence_after();
        // S <- S Diag(gamma_C) + Delta^T K~ (this thread's 64 columns), then its fp16 copy
        {
            const float* gam = reinterpret_cast<const float*>(S_ + kOffGam) + 64 * half;
            for (int q2 = 0; q2 < 2; ++q2) {
                float x[32];
                tmem_ld32(tD3 + lane_off + 64 * half + 32 * q2, x);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 32; ++e) s[32 * q2 + e] = fmaf(gam[32 * q2 + e], s[32 * q2 + e], x[e]);
            }
#pragma unroll
            for (int ci = 0; ci < 8; ++ci) st16(sS + kmajor_off(j, 64 * half + ci * 8, 128), pack8(s + ci * 8));
        }
        // O rows r in [32*half, 32*half + 32), column j
        {
            float x[32];
            tmem_ld32(tD1 + lane_off + 64 + 32 * half, x);
            tmem_ld_wait();
            const int r0 = c * kC + 32 * half;
#pragma unroll
            for (int e = 0; e < 32; ++e)
                if (r0 + e < T) store_f32(o + ((size_t)(b * T + r0 + e) * H + h) * dv + j, scale * x[e]);
        }
        tc_fence_before();
        __syncthreads();
        if (tid == 0 && c + 2 < NC) {
            fence_proxy_async_smem();
            mbar_arrive_expect_tx(&full[st], kHandoffBytes);
            bulk_g2s(S_, src + (size_t)(c + 2) * kHandoffStride, kHandoffBytes, &full[st]);
        }
    }
    if (S_T != nullptr) {
        float* dst = S_T + ((size_t)bh * kD + j) * kD + 64 * half;
#pragma unroll
        for (int e = 0; e < 64; e += 4) *reinterpret_cast<float4*>(dst + e) = make_float4(s[e], s[e + 1], s[e + 2], s[e + 3]);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem_base, 256);
}

template <int MODE>
cudaError_t launch_prep(const ChunkProblem& p, int NC, cudaStream_t stream) {
    auto kern = chunk_prep_kernel<MODE>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kPrepSmem);
    if (err != cudaSuccess) return err;
    dim3 grid(NC, p.H, p.B);
    kern<<<grid, kPrepThreads, kPrepSmem, stream>>>(
        static_cast<const __nv_bfloat16*>(p.q), static_cast<const __nv_bfloat16*>(p.k),
        static_cast<const __nv_bfloat16*>(p.v), p.g, p.beta, p.T, p.H, NC, static_cast<uint8_t*>(p.workspace),
        p.status);
    return cudaGetLastError();
}

template <typename Tout>
cudaError_t launch_state(const ChunkProblem& p, int NC, cudaStream_t stream) {
    auto kern = chunk_state_kernel<Tout>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kStateSmem);
    if (err != cudaSuccess) return err;
    kern<<<p.B * p.H, kStateThreads, kStateSmem, stream>>>(static_cast<const uint8_t*>(p.workspace), p.S0,
                                                          static_cast<Tout*>(p.o), p.S_T, p.T, p.H, NC, p.scale,
                                                          p.status);
    return cudaGetLastError();
}

}  // namespace

bool chunk_tc_supported(int dk, int dv, int chunk, int dtype, int o_dtype) {
    return dtype == GDR_BF16 && (o_dtype == GDR_F32 || o_dtype == GDR_BF16) && dk == kD && dv == kD && chunk == kC;
}

size_t chunk_tc_workspace_bytes(int B, int T, int H, int, int, int, int) {
    const size_t NC = (size_t)(T + kC - 1) / kC;
    return (size_t)B * H * NC * kHandoffStride;
}

int chunk_tc_launches(int, int, int, int, int, int, int) { return 2; }

cudaError_t launch_chunk_tc(const ChunkProblem& p, cudaStream_t stream) {
    const int NC = (p.T + kC - 1) / kC;
    cudaError_t err = cudaSuccess;
    switch (p.mode) {
        case GDR_DECAY_NONE: err = launch_prep<GDR_DECAY_NONE>(p, NC, stream); break;
        case GDR_DECAY_SCALAR: err = launch_prep<GDR_DECAY_SCALAR>(p, NC, stream); break;
        case GDR_DECAY_CHANNEL: err = launch_prep<GDR_DECAY_CHANNEL>(p, NC, stream); break;
        default: return cudaErrorInvalidValue;
    }
    if (err != cudaSuccess) return err;
    if (p.o_dtype == GDR_BF16) return launch_state<__nv_bfloat16>(p, NC, stream);
    return launch_state<float>(p, NC, stream);
}

}  // namespace gdr
