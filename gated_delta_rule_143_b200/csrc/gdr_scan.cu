// gdr_scan.cu -- sequence-parallel forward for few heads and long sequences (segment scan).
//
// The state evolves by an affine map per token, S_t = S_{t-1} A_t + B_t with A_t = Diag(alpha_t)
// (I - beta_t k_t k_t^T) and B_t = beta_t v_t k_t^T ("linear attention and its gated descendants",
// closing summary of the gated variants: a multiplicative transition plus a write, which composes
// associatively; the same page's Hardware Performance section asks for sequence-level parallelism
// when batch x heads is small). Splitting each sequence into s segments of equal length:
//
//   S_end(i)  = S_in(i) M(i) + S_end^0(i),   M(i) = prod of the A_t of segment i,
//   o_t       = o_t^0 + S_in(i) (scale * prod_{u <= t in segment i} A_u q_t)      (t in segment i)
//
// where ^0 marks the segment run from a zero state. Both parts come from the chunked forward on the
// [B*s, T/s, H] view of the same tensors, so every segment is an independent "sequence": one prep pass
// writes the hand-off blocks of every chunk, and one state-kernel launch runs over them
//   the data chains:       S0 = 0                    -> o^0 and S_end^0(i);
//   the transition chains: S0 = I, no write (U = 0)  -> O_I = scale * prod A q_t per token, S_T = M(i)
// (the transition of a chunk, Diag(gamma_C) - W^T K~, needs only the blocks' S-independent factors).
// Then the carry, S_in(0) = S0, S_in(i+1) = S_in(i) M(i) + S_end^0(i) (s steps per head, rows in
// parallel), and the correction o = o^0 + O_I S_in(i)^T on warp MMAs (tf32 operands, fp32
// accumulation). The chains are s times shorter than the sequence's and 2 s times as many run at once;
// the price is the transition chains and the correction's traffic.
#include "gdr_sm100.cuh"

namespace gdr {
namespace {

using namespace sm100;

constexpr int kSD = 128;  // d_k = d_v on this path

// One CTA per (8 state rows, head). Segment-head (b, i, h) has index (b * s + i) * H + h in the
// run-A/B state arrays. Writes S_in(i) for every segment and S_in(s) = S_T.
constexpr int kCarryRows = 8;
__global__ void __launch_bounds__(256)
scan_carry_kernel(const float* S0, const float* __restrict__ M, const float* __restrict__ Send,
                  float* __restrict__ Sin, float* S_T, int H, int s) {
    // S_T may be S0 (in-place carry): each element is read first and written last by the same thread
    extern __shared__ float carry_smem[];
    float* sM = carry_smem;                                                   // M(i), [m][c]
    auto sS = reinterpret_cast<float(*)[kSD]>(carry_smem + kSD * kSD);       // S_in rows of this CTA
    const int tid = threadIdx.x, lane = tid & 31, jr = tid >> 5;
    const int j = blockIdx.x * kCarryRows + jr;  // state row of this warp
    const int bh = blockIdx.y, b = bh / H, h = bh % H;
    float x[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) x[q] = S0 != nullptr ? S0[((size_t)bh * kSD + j) * kSD + lane + 32 * q] : 0.f;
    for (int i = 0; i < s; ++i) {
        const size_t sh = ((size_t)b * s + i) * H + h;
        __syncthreads();  // the previous step's readers of sM / sS are done
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            sS[jr][lane + 32 * q] = x[q];
            Sin[(sh * kSD + j) * kSD + lane + 32 * q] = x[q];
        }
        const float4* m4 = reinterpret_cast<const float4*>(M + sh * kSD * kSD);
        for (int e = tid; e < kSD * kSD / 4; e += 256) reinterpret_cast<float4*>(sM)[e] = m4[e];
        __syncthreads();
        float y[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) y[q] = Send[(sh * kSD + j) * kSD + lane + 32 * q];
#pragma unroll 8
        for (int m = 0; m < kSD; ++m) {
            const float a = sS[jr][m];
#pragma unroll
            for (int q = 0; q < 4; ++q) y[q] = fmaf(a, sM[m * kSD + lane + 32 * q], y[q]);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) x[q] = y[q];
    }
    if (S_T != nullptr) {
#pragma unroll
        for (int q = 0; q < 4; ++q) S_T[((size_t)bh * kSD + j) * kSD + lane + 32 * q] = x[q];
    }
}

// o[b, t, h, :] = o0[b, t, h, :] + O_I[b, t, h, :] S_in(b, i, h)^T for the tokens of segment i, on
// m16n8k8 tf32 warp MMAs. S_in sits in shared memory as tf32 (once per CTA); each warp takes 16-token
// tiles (all 128 output columns, 64 accumulators per thread) and reads its A fragments straight from
// global memory. The sum over k is order-free, so both operands use one permutation of each 8-wide k
// step: logical k = t and t + 4 of thread (g, t) are physical columns 2t and 2t + 1. A thread's two A
// values per row and its two B values are then adjacent (8-byte loads; a warp reads whole 32-byte
// sectors of O_I), and with a row stride of 136 words the B reads hit 32 distinct banks per half-warp.
constexpr int kLdB = kSD + 8;
constexpr int kCorrWarps = 8;
constexpr int kCorrTilesPerWarp = 4;  // 16-token tiles per warp
constexpr int kCorrRowsPerCta = kCorrWarps * kCorrTilesPerWarp * 16;  // 512 tokens

template <typename Tout>
__global__ void __launch_bounds__(kCorrWarps * 32, 2)
scan_correct_kernel(const float* o0, const float* __restrict__ OI, const float* __restrict__ Sin, Tout* o, int H,
                    int s, int Ts, bool has_s0) {
    // o0 may be o itself (fp32 output): each element is read, then written, by the same thread
    extern __shared__ uint32_t sBt[];  // S_in as tf32, [j][c] with row stride kLdB
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t4 = lane & 3;
    const int sh = blockIdx.y;  // (b * s + i) * H + h
    const int h = sh % H, bs = sh / H, i = bs % s;
    const bool correct = i > 0 || has_s0;
    if (!correct && static_cast<const void*>(o0) == static_cast<const void*>(o)) return;  // nothing to add
    if (correct) {
        const float4* src = reinterpret_cast<const float4*>(Sin + (size_t)sh * kSD * kSD);
        for (int e = tid; e < kSD * kSD / 4; e += kCorrWarps * 32) {
            const int j = e / (kSD / 4), c4 = e % (kSD / 4);
            const float4 v = src[e];
            *reinterpret_cast<uint4*>(sBt + j * kLdB + 4 * c4) = make_uint4(to_tf32(v.x), to_tf32(v.y), to_tf32(v.z),
                                                                             to_tf32(v.w));
        }
        __syncthreads();
    }
    for (int u = 0; u < kCorrTilesPerWarp; ++u) {
        const int t0 = blockIdx.x * kCorrRowsPerCta + (warp * kCorrTilesPerWarp + u) * 16;
        if (t0 >= Ts) break;
        const size_t rg = ((size_t)bs * Ts + t0 + g) * H + h;  // token row of fragment row g
        const size_t rg8 = rg + (size_t)8 * H;                  // and of row g + 8
        float acc[16][4];
#pragma unroll
        for (int n = 0; n < 16; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[n][e] = 0.f;
        if (correct) {
#pragma unroll
            for (int kh = 0; kh < 2; ++kh) {  // two halves of k: 8 k-steps of A in registers at a time
                float2 alo[8], ahi[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int col = 8 * (8 * kh + j) + 2 * t4;
                    alo[j] = __ldg(reinterpret_cast<const float2*>(OI + rg * kSD + col));
                    ahi[j] = __ldg(reinterpret_cast<const float2*>(OI + rg8 * kSD + col));
                }
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int col = 8 * (8 * kh + j) + 2 * t4;
                    const uint32_t a[4] = {to_tf32(alo[j].x), to_tf32(ahi[j].x), to_tf32(alo[j].y), to_tf32(ahi[j].y)};
#pragma unroll
                    for (int n = 0; n < 16; ++n) {
                        const uint2 bv = *reinterpret_cast<const uint2*>(sBt + (8 * n + g) * kLdB + col);
                        const uint32_t bb[2] = {bv.x, bv.y};
                        mma_tf32_16x8x8(acc[n], a, bb);
                    }
                }
            }
        }
        // epilogue: rows g and g + 8, columns 8 n + 2 t4 (+ 1). Every o0 load is issued before any
        // store (o0 may be o: with stores in between, each load would wait for the one before)
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const size_t row = half ? rg8 : rg;
#pragma unroll
            for (int n = 0; n < 16; ++n) {
                const float2 base = *reinterpret_cast<const float2*>(o0 + row * kSD + 8 * n + 2 * t4);
                acc[n][2 * half] += base.x;
                acc[n][2 * half + 1] += base.y;
            }
        }
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const size_t row = half ? rg8 : rg;
#pragma unroll
            for (int n = 0; n < 16; ++n) {
                const int col = 8 * n + 2 * t4;
                const float v0 = acc[n][2 * half], v1 = acc[n][2 * half + 1];
                if (sizeof(Tout) == 4) {
                    *reinterpret_cast<float2*>(reinterpret_cast<float*>(o) + row * kSD + col) = make_float2(v0, v1);
                } else {
                    *reinterpret_cast<__nv_bfloat162*>(reinterpret_cast<__nv_bfloat16*>(o) + row * kSD + col) =
                        __floats2bfloat162_rn(v0, v1);
                }
            }
        }
    }
}

size_t al256(size_t x) { return (x + 255) & ~size_t(255); }

struct ScanLayout {
    size_t run, oi, m, send, sin, o0, total;
};

ScanLayout scan_layout(int B, int T, int H, int mode, int n_seg, int o_dtype) {
    (void)mode;
    ScanLayout L{};
    const int Ts = T / n_seg;
    const size_t nsh = (size_t)B * n_seg * H, ntok = (size_t)B * T * H;
    size_t off = 0;
    L.run = off;   off += al256(chunk_tc_pair_workspace_bytes(B * n_seg, Ts, H));
    L.oi = off;    off += al256(ntok * kSD * 4);
    L.m = off;     off += al256(nsh * kSD * kSD * 4);
    L.send = off;  off += al256(nsh * kSD * kSD * 4);
    L.sin = off;   off += al256(nsh * kSD * kSD * 4);
    L.o0 = off;    off += o_dtype == GDR_F32 ? 0 : al256(ntok * kSD * 4);
    L.total = off;
    return L;
}

}  // namespace

bool scan_supported(int B, int T, int H, int dk, int dv, int chunk, int dtype, int o_dtype, int n_seg) {
    (void)B;
    (void)H;
    return chunk_tc_supported(dk, dv, chunk, dtype, o_dtype) && n_seg >= 2 && T % (n_seg * chunk) == 0;
}

size_t scan_workspace_bytes(int B, int T, int H, int mode, int n_seg, int o_dtype) {
    return scan_layout(B, T, H, mode, n_seg, o_dtype).total;
}

cudaError_t launch_scan(const ChunkProblem& p, int n_seg, cudaStream_t stream) {
    const ScanLayout L = scan_layout(p.B, p.T, p.H, p.mode, n_seg, p.o_dtype);
    uint8_t* ws = static_cast<uint8_t*>(p.workspace);
    const int Ts = p.T / n_seg, Bs = p.B * n_seg;
    const size_t nsh = (size_t)Bs * p.H;
    float* oi = reinterpret_cast<float*>(ws + L.oi);
    float* M = reinterpret_cast<float*>(ws + L.m);
    float* send = reinterpret_cast<float*>(ws + L.send);
    float* sin = reinterpret_cast<float*>(ws + L.sin);
    float* o0 = p.o_dtype == GDR_F32 ? static_cast<float*>(p.o) : reinterpret_cast<float*>(ws + L.o0);
    cudaError_t err;

    // every segment from a zero state, and every segment's transition, over one set of blocks
    ChunkProblem a = p;
    a.B = Bs;
    a.T = Ts;
    a.S0 = nullptr;
    a.o = o0;
    a.o_dtype = GDR_F32;
    a.S_T = send;
    a.workspace = ws + L.run;
    a.workspace_bytes = L.oi - L.run;
    if ((err = launch_chunk_tc_pair(a, oi, M, stream)) != cudaSuccess) return err;
    // carry the true incoming state across the segments
    const size_t carry_smem = (size_t)(kSD * kSD + kCarryRows * kSD) * sizeof(float);
    if ((err = cudaFuncSetAttribute(scan_carry_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)carry_smem)) !=
        cudaSuccess)
        return err;
    scan_carry_kernel<<<dim3(kSD / kCarryRows, p.B * p.H), 256, carry_smem, stream>>>(p.S0, M, send, sin, p.S_T, p.H,
                                                                                       n_seg);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    profile_after_launch(stream);
    // o = o^0 + O_I S_in^T
    const size_t smem = (size_t)kSD * kLdB * sizeof(uint32_t);
    const dim3 grid((Ts + kCorrRowsPerCta - 1) / kCorrRowsPerCta, (unsigned)nsh);
    if (p.o_dtype == GDR_BF16) {
        auto kern = scan_correct_kernel<__nv_bfloat16>;
        if ((err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
            return err;
        kern<<<grid, 256, smem, stream>>>(o0, oi, sin, static_cast<__nv_bfloat16*>(p.o), p.H, n_seg, Ts,
                                          p.S0 != nullptr);
    } else {
        auto kern = scan_correct_kernel<float>;
        if ((err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
            return err;
        kern<<<grid, 256, smem, stream>>>(o0, oi, sin, static_cast<float*>(p.o), p.H, n_seg, Ts, p.S0 != nullptr);
    }
    profile_after_launch(stream);
    return cudaGetLastError();
}

}  // namespace gdr
