// gdr_internal.cuh -- declarations shared by the library's CUDA translation units.
// Not installed; the public interface is include/gdr.h.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "gdr.h"

namespace gdr {

// Everything one chunked-forward launch needs. Pointers are device pointers.
struct ChunkProblem {
    const void* q;
    const void* k;
    const void* v;
    const float* g;
    const float* beta;
    const float* S0;
    void* o;
    float* S_T;
    int B, T, H, dk, dv, chunk, mode, dtype, o_dtype;
    void* workspace;
    size_t workspace_bytes;
    int* status;  // device status word (first error wins)
    float scale;
    int prologue;             // gdr_prologue flags: steps of the mixer layer done on the inputs in-kernel
    const float* gate_scale;  // [H] A of g = -A softplus(a) (GDR_PRO_GATE_SOFTPLUS), NULL = 1
    const float* erase;       // Gated DeltaNet-2: [B,T,H,d_k] erase gate (NULL: the delta rule with beta)
    const float* write;       // Gated DeltaNet-2: [B,T,H,d_v] write gate
};

struct DecodeProblem {
    const void* q;
    const void* k;
    const void* v;
    const float* g;
    const float* beta;
    float* S;
    void* o;
    int B, H, dk, dv, mode, dtype, o_dtype;
    int* status;
    float scale;
    int prologue;             // as ChunkProblem
    const float* gate_scale;
    const float* erase;       // Gated DeltaNet-2: [B,H,d_k] erase gate, NULL for the delta rule
    const float* write;       // Gated DeltaNet-2: [B,H,d_v] write gate
};

// Everything one backward call needs (gdr_chunk_bwd). Pointers are device pointers.
struct BwdProblem {
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
    void* workspace;
    int B, T, H, dk_dim, dv_dim, mode, dtype;
    float scale;
    int* status;  // device status word (a bounded wait that expired)
};

// The prologue's elementwise steps (gdr_prologue), in fp32 with CUDA's math functions.
__device__ __forceinline__ float pro_sigmoid(float x) { return 1.f / (1.f + expf(-x)); }
// g = -A softplus(a), softplus(a) = max(a, 0) + log(1 + e^-|a|)
__device__ __forceinline__ float pro_gate(float a, float A) { return -A * (fmaxf(a, 0.f) + log1pf(expf(-fabsf(a)))); }
// 1 / |x| from the sum of squares; an all-zero vector (or one whose squares underflow) stays zero
__device__ __forceinline__ float pro_inv_norm(float sum_sq) { return sum_sq > 0.f ? rsqrtf(sum_sq) : 0.f; }

// Device status codes written by kernels (mirror gdr_status).
constexpr int kStatusTimeout = GDR_ERR_TIMEOUT;

__device__ __forceinline__ void report_status(int* status, int code) {
    if (status != nullptr) atomicCAS(status, 0, code);
}

// The status record: [0] the code; for the first expired wait also [1] which wait (1: mbarrier,
// 2: mbarrier with abort, 3: global flag), [2] blockIdx.x, [3] threadIdx.x, [4] the barrier's shared
// address and parity (addr | parity << 31) or the flag's target. gdr_sync_status reports and clears it.
constexpr int kStatusWords = 8;
__device__ __forceinline__ void report_timeout(int* status, int site, int detail) {
    if (status != nullptr && atomicCAS(status, 0, kStatusTimeout) == 0) {
        status[1] = site;
        status[2] = (int)blockIdx.x;
        status[3] = (int)threadIdx.x;
        status[4] = detail;
        __threadfence();
    }
}

template <typename T>
__device__ __forceinline__ float load_f32(const T* p);
template <>
__device__ __forceinline__ float load_f32<float>(const float* p) { return *p; }
template <>
__device__ __forceinline__ float load_f32<__nv_bfloat16>(const __nv_bfloat16* p) {
    return __bfloat162float(*p);
}

template <typename T>
__device__ __forceinline__ void store_f32(T* p, float x);
template <>
__device__ __forceinline__ void store_f32<float>(float* p, float x) { *p = x; }
template <>
__device__ __forceinline__ void store_f32<__nv_bfloat16>(__nv_bfloat16* p, float x) {
    *p = __float2bfloat16_rn(x);
}

// CUDA-core fp32 chunked forward (any supported shape, fp32 or bf16 inputs).
bool chunk_simt_supported(int dk, int dv, int chunk);
// Records the next caller-supplied profiling event (gdr_profile_next_call) on `stream`, if one is
// pending for the chunked forward in progress on this host thread. Launchers call it right after
// each kernel launch.
void profile_after_launch(cudaStream_t stream);

cudaError_t launch_chunk_simt(const ChunkProblem& p, cudaStream_t stream);

// Tensor-core (tcgen05) chunked forward: bf16, d_k = d_v = 128, chunk = 64.
bool chunk_tc_supported(int dk, int dv, int chunk, int dtype, int o_dtype);
// ew: Gated DeltaNet-2 (erase / write gates: the two-pass plan)
size_t chunk_tc_workspace_bytes(int B, int T, int H, int dk, int dv, int chunk, int mode, bool ew = false);
cudaError_t launch_chunk_tc(const ChunkProblem& p, cudaStream_t stream);
int chunk_tc_launches(int B, int T, int H, int dk, int dv, int chunk, int mode);
int chunk_tc_plan(int B, int T, int H, int dk, int dv, int chunk, int mode, int* precomputed_chunks);

// The prep pass and a state kernel running both the data chains and, over the same blocks, the
// transition chains (identity state, no write) of every head; outputs fp32 (segment scan).
size_t chunk_tc_pair_workspace_bytes(int B, int T, int H);
cudaError_t launch_chunk_tc_pair(const ChunkProblem& p, void* o2, float* S_T2, cudaStream_t stream);

// Segment scan (sequence-parallel forward) on the tensor-core path: the chunked forward on the
// [B * n_seg, T / n_seg, H] view twice (data from a zero state; identity state with v = 0), a carry
// of the incoming states across the segments and a tensor-core correction of the outputs.
bool scan_supported(int B, int T, int H, int dk, int dv, int chunk, int dtype, int o_dtype, int n_seg);
size_t scan_workspace_bytes(int B, int T, int H, int mode, int n_seg, int o_dtype);
cudaError_t launch_scan(const ChunkProblem& p, int n_seg, cudaStream_t stream);

// Self-test of the bounded waits (gdr_selftest_bounded_wait): one CTA whose roles wait on a flag
// that nothing sets, with a wait bound of limit_ns; then the time it ran, read after the stream.
cudaError_t launch_bounded_wait_selftest(int* status, uint64_t limit_ns, cudaStream_t stream);
cudaError_t read_bounded_wait_selftest_elapsed(unsigned long long* elapsed_ns);

// Backward of the forward (fp32 CUDA cores): state history, then the reverse sweep.
bool bwd_supported(int dk, int dv);
size_t bwd_workspace_bytes(int B, int T, int H, int dk, int dv);
cudaError_t launch_bwd(const BwdProblem& p, cudaStream_t stream);

// Bandwidth-bound decode step.
bool decode_supported(int dk, int dv);
cudaError_t launch_decode(const DecodeProblem& p, cudaStream_t stream);

}  // namespace gdr
