// gdr_api.cu -- the library's C ABI (declared in include/gdr.h): argument validation, the
// per-device status word and dispatch to the kernels. No entry point allocates device memory.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <mutex>

#include "gdr_internal.cuh"

namespace gdr {
namespace {

thread_local char g_last_error[512] = "";

int fail(int code, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
    va_end(ap);
    return code;
}

int ok() {
    g_last_error[0] = '\0';
    return GDR_OK;
}

// Per-kernel timing events for the next chunked forward on this thread (gdr_profile_next_call).
// `pending` is set by the caller; the outermost chunk-forward entry point moves it to `active`
// for the duration of the call and clears both on exit.
struct ProfileEvents {
    cudaEvent_t ev[8];
    int n = 0, next = 0;
};
thread_local ProfileEvents g_prof_pending, g_prof_active;
thread_local int g_prof_depth = 0;

struct ProfileScope {
    ProfileScope() {
        if (g_prof_depth++ == 0) {
            g_prof_active = g_prof_pending;
            g_prof_active.next = 0;
            g_prof_pending.n = 0;
        }
    }
    ~ProfileScope() {
        if (--g_prof_depth == 0) g_prof_active.n = 0;
    }
};

// Device status record: kernels record the first device-side error here (a bounded wait that
// expired, with where it happened). A statically sized __device__ array, so it needs no
// allocation; each device that loads the library has its own copy. Host code reaches it through
// its address.
__device__ int g_status_word[kStatusWords] = {};

constexpr int kMaxDevices = 64;
std::mutex g_dev_mutex;
int* g_status_ptr[kMaxDevices] = {};
int g_dev_major[kMaxDevices] = {};

// Resolves (once per device) the status word's device address and the compute capability.
int device_setup(int** status, int* major) {
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return fail(GDR_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(err));
    if (dev < 0 || dev >= kMaxDevices) return fail(GDR_ERR_DEVICE, "device ordinal %d out of range", dev);
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    if (g_status_ptr[dev] == nullptr) {
        int maj = 0;
        err = cudaDeviceGetAttribute(&maj, cudaDevAttrComputeCapabilityMajor, dev);
        if (err != cudaSuccess) return fail(GDR_ERR_CUDA, "cudaDeviceGetAttribute: %s", cudaGetErrorString(err));
        void* p = nullptr;
        err = cudaGetSymbolAddress(&p, g_status_word);
        if (err != cudaSuccess) return fail(GDR_ERR_CUDA, "cudaGetSymbolAddress(status): %s", cudaGetErrorString(err));
        g_dev_major[dev] = maj;
        g_status_ptr[dev] = static_cast<int*>(p);
    }
    *status = g_status_ptr[dev];
    *major = g_dev_major[dev];
    return GDR_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlap(const void* a, size_t na, const void* b, size_t nb) {
    if (a == nullptr || b == nullptr || na == 0 || nb == 0) return false;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + nb && b0 < a0 + na;
}

size_t elem_bytes(int dtype) { return dtype == GDR_BF16 ? 2 : 4; }

int check_enums(int mode, int dtype, int o_dtype) {
    if (mode != GDR_DECAY_NONE && mode != GDR_DECAY_SCALAR && mode != GDR_DECAY_CHANNEL)
        return fail(GDR_ERR_INVALID_ARG, "unknown decay mode %d", mode);
    if (dtype != GDR_F32 && dtype != GDR_BF16) return fail(GDR_ERR_INVALID_ARG, "unknown dtype %d", dtype);
    if (o_dtype != GDR_F32 && o_dtype != GDR_BF16) return fail(GDR_ERR_INVALID_ARG, "unknown o_dtype %d", o_dtype);
    if (dtype == GDR_F32 && o_dtype == GDR_BF16)
        return fail(GDR_ERR_UNSUPPORTED, "fp32 inputs with a bf16 output are not supported");
    return GDR_OK;
}

int chunk_shape_check(int B, int T, int H, int dk, int dv, int chunk, int mode, int dtype, int o_dtype) {
    if (int rc = check_enums(mode, dtype, o_dtype)) return rc;
    if (B <= 0 || T <= 0 || H <= 0 || dk <= 0 || dv <= 0 || chunk <= 0)
        return fail(GDR_ERR_INVALID_ARG, "sizes must be positive (B=%d T=%d H=%d d_k=%d d_v=%d chunk=%d)", B, T, H,
                    dk, dv, chunk);
    if (H > 65535 || B > 65535) return fail(GDR_ERR_UNSUPPORTED, "B and H must be <= 65535");
    if (!chunk_tc_supported(dk, dv, chunk, dtype, o_dtype) && !chunk_simt_supported(dk, dv, chunk))
        return fail(GDR_ERR_UNSUPPORTED,
                    "unsupported shape d_k=%d d_v=%d chunk=%d (supported: chunk 64 with d_k, d_v in {32, 64, 128})",
                    dk, dv, chunk);
    return GDR_OK;
}

int prologue_check(int prologue, int mode) {
    const int all = GDR_PRO_L2NORM_QK | GDR_PRO_BETA_SIGMOID | GDR_PRO_GATE_SOFTPLUS;
    if (prologue & ~all) return fail(GDR_ERR_INVALID_ARG, "unknown prologue flags 0x%x", prologue & ~all);
    if ((prologue & GDR_PRO_GATE_SOFTPLUS) && mode == GDR_DECAY_NONE)
        return fail(GDR_ERR_INVALID_ARG, "GDR_PRO_GATE_SOFTPLUS needs a gated decay mode");
    return GDR_OK;
}

// Segments gdr_chunk_fwd gives a problem on its own: few heads and long sequences, where one serial
// chain per head leaves most SMs idle. The data and transition chains of B * H * s segment-heads
// should about fill the GPU (2 B H s <= 128) while the carry's s sequential steps stay short (s <= 16)
// and every segment keeps at least 16 chunks. Measured at T = 65536 (fused plan: about 2.3 ms):
// 2 heads 362 us with 16 segments, 4 heads 480 us (16), 8 heads 751 us (8), 16 heads 1.32 ms (4);
// 16 heads at T = 16384: 411 us with 4 segments against 606 us fused. 0: no segment scan.
int auto_segments(int B, int T, int H, int dk, int dv, int chunk, int dtype, int o_dtype) {
    const size_t BH = (size_t)B * H;
    const int NC = (T + chunk - 1) / chunk;
    if (BH > 16 || NC < 256) return 0;
    int s = 16;
    while (s > 2 && (BH * s > 64 || NC / s < 16 || T % (s * chunk) != 0)) s >>= 1;
    return scan_supported(B, T, H, dk, dv, chunk, dtype, o_dtype, s) ? s : 0;
}

// Gated DeltaNet-2 runs on the tensor cores for the channel decay at the tensor-core shapes (the
// channel gate's plans), on the CUDA cores otherwise.
bool gdn2_on_tc(int dk, int dv, int chunk, int mode, int dtype, int o_dtype) {
    return mode == GDR_DECAY_CHANNEL && chunk_tc_supported(dk, dv, chunk, dtype, o_dtype);
}

// The chunked forward behind gdr_chunk_fwd(_ex, _scan, _noalloc) and gdr_chunk_fwd_gdn2. n_seg: 0 = the
// plan chosen from the shape (auto_segments), -1 = no segment scan, >= 2 = that many segments. With
// erase / write (Gated DeltaNet-2) beta is unused, and there is no prologue or segment scan.
int chunk_fwd_impl(const void* q, const void* k, const void* v, const float* g, const float* beta, const float* S0,
                   void* o, float* S_T, int B, int T, int H, int dk, int dv, int chunk, int mode, int dtype,
                   int o_dtype, int prologue, const float* gate_scale, int n_seg, const float* erase,
                   const float* write, void* workspace, size_t workspace_bytes, void* stream) {
    ProfileScope prof_scope;
    if (int rc = chunk_shape_check(B, T, H, dk, dv, chunk, mode, dtype, o_dtype)) return rc;
    const bool ew = erase != nullptr || write != nullptr;
    if (ew) {
        n_seg = -1;
        beta = nullptr;
        if (!erase || !write) return fail(GDR_ERR_INVALID_ARG, "erase and write must both be non-null");
        if (!gdn2_on_tc(dk, dv, chunk, mode, dtype, o_dtype) && !chunk_simt_supported(dk, dv, chunk))
            return fail(GDR_ERR_UNSUPPORTED,
                        "Gated DeltaNet-2: d_k, d_v in {32, 64, 128} and chunk 64 (got %d, %d, %d)", dk, dv, chunk);
    }
    if (n_seg == 0) n_seg = auto_segments(B, T, H, dk, dv, chunk, dtype, o_dtype);
    if (n_seg < 0) n_seg = 0;
    if (n_seg != 0 && !scan_supported(B, T, H, dk, dv, chunk, dtype, o_dtype, n_seg))
        return fail(GDR_ERR_UNSUPPORTED,
                    "segment scan: bf16 q/k/v, d_k = d_v = 128, chunk 64, n_seg >= 2 and T a multiple of "
                    "n_seg * chunk (got T=%d, n_seg=%d)", T, n_seg);
    if (int rc = prologue_check(prologue, mode)) return rc;
    if (!(prologue & GDR_PRO_GATE_SOFTPLUS)) gate_scale = nullptr;
    if (!q || !k || !v || (!beta && !ew) || !o)
        return fail(GDR_ERR_INVALID_ARG, "q, k, v, beta and o must be non-null");
    if (mode != GDR_DECAY_NONE && !g) return fail(GDR_ERR_INVALID_ARG, "g must be non-null for a gated decay mode");
    if (mode == GDR_DECAY_NONE) g = nullptr;
    const void* ptrs[] = {q, k, v, g, beta, S0, o, S_T, workspace, gate_scale, erase, write};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return fail(GDR_ERR_MISALIGNED, "pointer %p is not 16-byte aligned", p);
    const size_t ntok = (size_t)B * T * H;
    const size_t eb = elem_bytes(dtype);
    const size_t bq = ntok * dk * eb, bv = ntok * dv * eb, bb = ntok * sizeof(float);
    const size_t bo = ntok * dv * elem_bytes(o_dtype);
    const size_t bg = mode == GDR_DECAY_NONE ? 0 : (mode == GDR_DECAY_SCALAR ? bb : ntok * dk * sizeof(float));
    const size_t bs = (size_t)B * H * dv * dk * sizeof(float);
    struct Span { const void* p; size_t n; const char* name; };
    const Span ins[] = {{q, bq, "q"}, {k, bq, "k"}, {v, bv, "v"}, {g, bg, "g"}, {beta, bb, "beta"}, {S0, bs, "S0"},
                        {gate_scale, H * sizeof(float), "gate_scale"}, {erase, ntok * dk * sizeof(float), "erase"},
                        {write, ntok * dv * sizeof(float), "write"}};
    for (const Span& s : ins) {
        if (overlap(o, bo, s.p, s.n)) return fail(GDR_ERR_INVALID_ARG, "o overlaps input %s", s.name);
        if (S_T != S0 && overlap(S_T, bs, s.p, s.n))
            return fail(GDR_ERR_INVALID_ARG, "S_T overlaps input %s (only S_T == S0 is allowed)", s.name);
    }
    if (overlap(o, bo, S_T, bs)) return fail(GDR_ERR_INVALID_ARG, "o overlaps S_T");
    const bool use_tc = ew ? gdn2_on_tc(dk, dv, chunk, mode, dtype, o_dtype)
                           : chunk_tc_supported(dk, dv, chunk, dtype, o_dtype);
    const size_t need = n_seg != 0 ? scan_workspace_bytes(B, T, H, mode, n_seg, o_dtype)
                                   : (use_tc ? chunk_tc_workspace_bytes(B, T, H, dk, dv, chunk, mode, ew) : 0);
    if (need > 0 && (workspace == nullptr || workspace_bytes < need))
        return fail(GDR_ERR_WORKSPACE, "workspace of %zu bytes required (got %zu at %p)", need, workspace_bytes,
                    workspace);
    if (need > 0) {
        for (const Span& s : ins)
            if (overlap(workspace, need, s.p, s.n)) return fail(GDR_ERR_INVALID_ARG, "workspace overlaps %s", s.name);
        if (overlap(workspace, need, o, bo) || overlap(workspace, need, S_T, bs))
            return fail(GDR_ERR_INVALID_ARG, "workspace overlaps an output");
    }
    int* status = nullptr;
    int major = 0;
    if (int rc = device_setup(&status, &major)) return rc;
    if (major != 10) return fail(GDR_ERR_DEVICE, "compute capability %d.x: this library is built for sm_100a", major);

    ChunkProblem p{q, k, v, g, beta, S0, o, S_T, B, T, H, dk, dv, chunk, mode, dtype, o_dtype, workspace,
                   workspace_bytes, status, (float)(1.0 / sqrt((double)dk)), prologue, gate_scale, erase, write};
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const cudaError_t err = n_seg != 0 ? launch_scan(p, n_seg, s) : (use_tc ? launch_chunk_tc(p, s) : launch_chunk_simt(p, s));
    if (err != cudaSuccess)
        return fail(GDR_ERR_CUDA, "%s chunk launch: %s", n_seg ? "segment-scan" : (use_tc ? "tensor-core" : "fp32"),
                    cudaGetErrorString(err));
    return ok();
}


// The decode step behind gdr_decode_step(_ex) and gdr_decode_step_gdn2 (erase / write in place of beta,
// no prologue).
int decode_impl(const void* q, const void* k, const void* v, const float* g, const float* beta, float* S, void* o,
                int B, int H, int dk, int dv, int mode, int dtype, int o_dtype, int prologue, const float* gate_scale,
                const float* erase, const float* write, void* stream) {
    if (int rc = check_enums(mode, dtype, o_dtype)) return rc;
    const bool ew = erase != nullptr || write != nullptr;
    if (ew && (!erase || !write)) return fail(GDR_ERR_INVALID_ARG, "erase and write must both be non-null");
    if (ew) beta = nullptr, prologue = GDR_PRO_NONE;
    if (int rc = prologue_check(prologue, mode)) return rc;
    if (!(prologue & GDR_PRO_GATE_SOFTPLUS)) gate_scale = nullptr;
    if (B <= 0 || H <= 0 || dk <= 0 || dv <= 0)
        return fail(GDR_ERR_INVALID_ARG, "sizes must be positive (B=%d H=%d d_k=%d d_v=%d)", B, H, dk, dv);
    if ((size_t)B * H > 0x7fffffffu) return fail(GDR_ERR_UNSUPPORTED, "B*H too large");
    if (!decode_supported(dk, dv))
        return fail(GDR_ERR_UNSUPPORTED, "unsupported d_k=%d (supported: 32, 64, 128, 256)", dk);
    if (!q || !k || !v || (!beta && !ew) || !S || !o)
        return fail(GDR_ERR_INVALID_ARG, "q, k, v, beta, S and o must be non-null");
    if (mode != GDR_DECAY_NONE && !g) return fail(GDR_ERR_INVALID_ARG, "g must be non-null for a gated decay mode");
    if (mode == GDR_DECAY_NONE) g = nullptr;
    const void* ptrs[] = {q, k, v, g, beta, S, o, gate_scale, erase, write};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return fail(GDR_ERR_MISALIGNED, "pointer %p is not 16-byte aligned", p);
    const size_t nh = (size_t)B * H, eb = elem_bytes(dtype);
    const size_t bs = nh * dv * dk * sizeof(float), bo = nh * dv * elem_bytes(o_dtype);
    struct Span { const void* p; size_t n; const char* name; };
    const Span ins[] = {{q, nh * dk * eb, "q"}, {k, nh * dk * eb, "k"}, {v, nh * dv * eb, "v"},
                        {mode == GDR_DECAY_NONE ? nullptr : g,
                         mode == GDR_DECAY_CHANNEL ? nh * dk * sizeof(float) : nh * sizeof(float), "g"},
                        {beta, nh * sizeof(float), "beta"}, {gate_scale, H * sizeof(float), "gate_scale"},
                        {erase, nh * dk * sizeof(float), "erase"}, {write, nh * dv * sizeof(float), "write"}};
    for (const Span& s : ins) {
        if (overlap(S, bs, s.p, s.n)) return fail(GDR_ERR_INVALID_ARG, "S overlaps input %s", s.name);
        if (overlap(o, bo, s.p, s.n)) return fail(GDR_ERR_INVALID_ARG, "o overlaps input %s", s.name);
    }
    if (overlap(o, bo, S, bs)) return fail(GDR_ERR_INVALID_ARG, "o overlaps S");
    int* status = nullptr;
    int major = 0;
    if (int rc = device_setup(&status, &major)) return rc;
    if (major != 10) return fail(GDR_ERR_DEVICE, "compute capability %d.x: this library is built for sm_100a", major);
    DecodeProblem p{q, k, v, mode == GDR_DECAY_NONE ? nullptr : g, beta, S, o, B, H, dk, dv, mode, dtype, o_dtype,
                    status, (float)(1.0 / sqrt((double)dk)), prologue, gate_scale, erase, write};
    const cudaError_t err = launch_decode(p, static_cast<cudaStream_t>(stream));
    if (err != cudaSuccess) return fail(GDR_ERR_CUDA, "decode launch: %s", cudaGetErrorString(err));
    return ok();
}

}  // namespace

void profile_after_launch(cudaStream_t stream) {
    if (g_prof_active.next < g_prof_active.n) cudaEventRecord(g_prof_active.ev[g_prof_active.next++], stream);
}

}  // namespace gdr

using namespace gdr;

extern "C" {

int gdr_version(void) { return 100; }

int gdr_profile_next_call(void* const* events, int n_events) {
    if (n_events < 0 || n_events > 8) return fail(GDR_ERR_INVALID_ARG, "n_events = %d (0 .. 8)", n_events);
    if (n_events > 0 && events == nullptr) return fail(GDR_ERR_INVALID_ARG, "events is NULL");
    for (int i = 0; i < n_events; ++i) g_prof_pending.ev[i] = static_cast<cudaEvent_t>(events[i]);
    g_prof_pending.n = n_events;
    return ok();
}

const char* gdr_last_error(void) { return g_last_error; }

size_t gdr_chunk_fwd_workspace_bytes(int B, int T, int H, int dk, int dv, int chunk, int mode, int dtype,
                                     int o_dtype) {
    char saved[sizeof(g_last_error)];
    memcpy(saved, g_last_error, sizeof(saved));
    const int rc = chunk_shape_check(B, T, H, dk, dv, chunk, mode, dtype, o_dtype);
    memcpy(g_last_error, saved, sizeof(saved));
    if (rc != GDR_OK) return 0;
    if (const int ns = auto_segments(B, T, H, dk, dv, chunk, dtype, o_dtype)) return scan_workspace_bytes(B, T, H, mode, ns, o_dtype);
    if (chunk_tc_supported(dk, dv, chunk, dtype, o_dtype)) return chunk_tc_workspace_bytes(B, T, H, dk, dv, chunk, mode);
    return 0;
}

int gdr_chunk_fwd_plan(int B, int T, int H, int dk, int dv, int chunk, int mode, int dtype, int o_dtype,
                       int* precomputed_chunks) {
    char saved[sizeof(g_last_error)];
    memcpy(saved, g_last_error, sizeof(saved));
    const int rc = chunk_shape_check(B, T, H, dk, dv, chunk, mode, dtype, o_dtype);
    memcpy(g_last_error, saved, sizeof(saved));
    if (precomputed_chunks != nullptr) *precomputed_chunks = 0;
    if (rc != GDR_OK) return GDR_PLAN_INVALID;
    if (!chunk_tc_supported(dk, dv, chunk, dtype, o_dtype)) return GDR_PLAN_CUDA_CORE;
    if (const int ns = auto_segments(B, T, H, dk, dv, chunk, dtype, o_dtype)) {
        if (precomputed_chunks != nullptr) *precomputed_chunks = ns;
        return GDR_PLAN_SCAN;
    }
    return chunk_tc_plan(B, T, H, dk, dv, chunk, mode, precomputed_chunks);
}

int gdr_chunk_fwd_launches(int B, int T, int H, int dk, int dv, int chunk, int mode, int dtype, int o_dtype) {
    char saved[sizeof(g_last_error)];
    memcpy(saved, g_last_error, sizeof(saved));
    const int rc = chunk_shape_check(B, T, H, dk, dv, chunk, mode, dtype, o_dtype);
    memcpy(g_last_error, saved, sizeof(saved));
    if (rc != GDR_OK) return 0;
    if (auto_segments(B, T, H, dk, dv, chunk, dtype, o_dtype)) return 4;  // prep, state, carry, correction
    return chunk_tc_supported(dk, dv, chunk, dtype, o_dtype) ? chunk_tc_launches(B, T, H, dk, dv, chunk, mode) : 1;
}

int gdr_chunk_fwd_ex(const void* q, const void* k, const void* v, const float* g, const float* beta,
                     const float* S0, void* o, float* S_T, int B, int T, int H, int dk, int dv, int chunk,
                     int mode, int dtype, int o_dtype, int prologue, const float* gate_scale, void* workspace,
                     size_t workspace_bytes, void* stream) {
    return chunk_fwd_impl(q, k, v, g, beta, S0, o, S_T, B, T, H, dk, dv, chunk, mode, dtype, o_dtype, prologue,
                          gate_scale, 0, nullptr, nullptr, workspace, workspace_bytes, stream);
}

int gdr_chunk_fwd_scan(const void* q, const void* k, const void* v, const float* g, const float* beta,
                       const float* S0, void* o, float* S_T, int B, int T, int H, int dk, int dv, int chunk,
                       int mode, int dtype, int o_dtype, int n_seg, void* workspace, size_t workspace_bytes,
                       void* stream) {
    if (n_seg < 2) return fail(GDR_ERR_INVALID_ARG, "n_seg = %d (at least 2)", n_seg);
    return chunk_fwd_impl(q, k, v, g, beta, S0, o, S_T, B, T, H, dk, dv, chunk, mode, dtype, o_dtype, GDR_PRO_NONE,
                          nullptr, n_seg, nullptr, nullptr, workspace, workspace_bytes, stream);
}

size_t gdr_chunk_fwd_scan_workspace_bytes(int B, int T, int H, int dk, int dv, int chunk, int mode, int dtype,
                                          int o_dtype, int n_seg) {
    char saved[sizeof(g_last_error)];
    memcpy(saved, g_last_error, sizeof(saved));
    const int rc = chunk_shape_check(B, T, H, dk, dv, chunk, mode, dtype, o_dtype);
    memcpy(g_last_error, saved, sizeof(saved));
    if (rc != GDR_OK || !scan_supported(B, T, H, dk, dv, chunk, dtype, o_dtype, n_seg)) return 0;
    return scan_workspace_bytes(B, T, H, mode, n_seg, o_dtype);
}

int gdr_chunk_fwd(const void* q, const void* k, const void* v, const float* g, const float* beta,
                  const float* S0, void* o, float* S_T, int B, int T, int H, int dk, int dv, int chunk,
                  int mode, int dtype, int o_dtype, void* workspace, size_t workspace_bytes, void* stream) {
    return gdr_chunk_fwd_ex(q, k, v, g, beta, S0, o, S_T, B, T, H, dk, dv, chunk, mode, dtype, o_dtype, GDR_PRO_NONE,
                            nullptr, workspace, workspace_bytes, stream);
}

int gdr_decode_step_ex(const void* q, const void* k, const void* v, const float* g, const float* beta, float* S,
                       void* o, int B, int H, int dk, int dv, int mode, int dtype, int o_dtype, int prologue,
                       const float* gate_scale, void* stream) {
    return decode_impl(q, k, v, g, beta, S, o, B, H, dk, dv, mode, dtype, o_dtype, prologue, gate_scale, nullptr,
                       nullptr, stream);
}

int gdr_decode_step(const void* q, const void* k, const void* v, const float* g, const float* beta, float* S,
                    void* o, int B, int H, int dk, int dv, int mode, int dtype, int o_dtype, void* stream) {
    return gdr_decode_step_ex(q, k, v, g, beta, S, o, B, H, dk, dv, mode, dtype, o_dtype, GDR_PRO_NONE, nullptr,
                              stream);
}

size_t gdr_chunk_fwd_gdn2_workspace_bytes(int B, int T, int H, int dk, int dv, int chunk, int mode, int dtype,
                                          int o_dtype) {
    char saved[sizeof(g_last_error)];
    memcpy(saved, g_last_error, sizeof(saved));
    const int rc = chunk_shape_check(B, T, H, dk, dv, chunk, mode, dtype, o_dtype);
    memcpy(g_last_error, saved, sizeof(saved));
    if (rc != GDR_OK || !gdn2_on_tc(dk, dv, chunk, mode, dtype, o_dtype)) return 0;
    return chunk_tc_workspace_bytes(B, T, H, dk, dv, chunk, mode, true);
}

int gdr_chunk_fwd_gdn2(const void* q, const void* k, const void* v, const float* g, const float* erase,
                       const float* write, const float* S0, void* o, float* S_T, int B, int T, int H, int dk, int dv,
                       int chunk, int mode, int dtype, int o_dtype, void* workspace, size_t workspace_bytes,
                       void* stream) {
    if (!erase || !write) return fail(GDR_ERR_INVALID_ARG, "erase and write must both be non-null");
    return chunk_fwd_impl(q, k, v, g, nullptr, S0, o, S_T, B, T, H, dk, dv, chunk, mode, dtype, o_dtype, GDR_PRO_NONE,
                          nullptr, -1, erase, write, workspace, workspace_bytes, stream);
}

int gdr_decode_step_gdn2(const void* q, const void* k, const void* v, const float* g, const float* erase,
                         const float* write, float* S, void* o, int B, int H, int dk, int dv, int mode, int dtype,
                         int o_dtype, void* stream) {
    if (!erase || !write) return fail(GDR_ERR_INVALID_ARG, "erase and write must both be non-null");
    return decode_impl(q, k, v, g, nullptr, S, o, B, H, dk, dv, mode, dtype, o_dtype, GDR_PRO_NONE, nullptr, erase,
                       write, stream);
}

size_t gdr_chunk_bwd_workspace_bytes(int B, int T, int H, int dk, int dv, int mode, int dtype) {
    if (B <= 0 || T <= 0 || H <= 0 || !bwd_supported(dk, dv)) return 0;
    if (mode != GDR_DECAY_NONE && mode != GDR_DECAY_SCALAR && mode != GDR_DECAY_CHANNEL) return 0;
    if (dtype != GDR_F32 && dtype != GDR_BF16) return 0;
    return bwd_workspace_bytes(B, T, H, dk, dv);
}

int gdr_chunk_bwd(const void* q, const void* k, const void* v, const float* g, const float* beta, const float* S0,
                  const void* dO, const float* dS_T, float* dq, float* dk_out, float* dv_out, float* dg,
                  float* dbeta, float* dS0, int B, int T, int H, int dk, int dv, int mode, int dtype,
                  void* workspace, size_t workspace_bytes, void* stream) {
    ProfileScope prof_scope;
    if (mode != GDR_DECAY_NONE && mode != GDR_DECAY_SCALAR && mode != GDR_DECAY_CHANNEL)
        return fail(GDR_ERR_INVALID_ARG, "unknown decay mode %d", mode);
    if (dtype != GDR_F32 && dtype != GDR_BF16) return fail(GDR_ERR_INVALID_ARG, "unknown dtype %d", dtype);
    if (B <= 0 || T <= 0 || H <= 0 || dk <= 0 || dv <= 0)
        return fail(GDR_ERR_INVALID_ARG, "sizes must be positive (B=%d T=%d H=%d d_k=%d d_v=%d)", B, T, H, dk, dv);
    if (H > 65535 || (size_t)B * H > 0x7fffffffu) return fail(GDR_ERR_UNSUPPORTED, "B * H too large");
    if (!bwd_supported(dk, dv))
        return fail(GDR_ERR_UNSUPPORTED, "unsupported d_k=%d d_v=%d (supported: 32, 64, 128 each)", dk, dv);
    if (!q || !k || !v || !beta || !dO || !dq || !dk_out || !dv_out || !dbeta)
        return fail(GDR_ERR_INVALID_ARG, "q, k, v, beta, dO, dq, dk, dv and dbeta must be non-null");
    if (mode != GDR_DECAY_NONE && (!g || !dg))
        return fail(GDR_ERR_INVALID_ARG, "g and dg must be non-null for a gated decay mode");
    if (mode == GDR_DECAY_NONE) g = nullptr, dg = nullptr;
    const void* ptrs[] = {q, k, v, g, beta, S0, dO, dS_T, dq, dk_out, dv_out, dg, dbeta, dS0, workspace};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return fail(GDR_ERR_MISALIGNED, "pointer %p is not 16-byte aligned", p);
    const size_t ntok = (size_t)B * T * H, eb = elem_bytes(dtype);
    const size_t bs = (size_t)B * H * dv * dk * sizeof(float);
    const size_t bgd = mode == GDR_DECAY_CHANNEL ? ntok * dk * sizeof(float) : ntok * sizeof(float);
    struct Span { const void* p; size_t n; const char* name; };
    const Span ins[] = {{q, ntok * dk * eb, "q"}, {k, ntok * dk * eb, "k"}, {v, ntok * dv * eb, "v"},
                        {g, bgd, "g"}, {beta, ntok * sizeof(float), "beta"}, {S0, bs, "S0"},
                        {dO, ntok * dv * eb, "dO"}, {dS_T, bs, "dS_T"}};
    const Span outs[] = {{dq, ntok * dk * sizeof(float), "dq"}, {dk_out, ntok * dk * sizeof(float), "dk"},
                         {dv_out, ntok * dv * sizeof(float), "dv"}, {dg, bgd, "dg"},
                         {dbeta, ntok * sizeof(float), "dbeta"}, {dS0, bs, "dS0"}};
    const size_t need = bwd_workspace_bytes(B, T, H, dk, dv);
    if (workspace == nullptr || workspace_bytes < need)
        return fail(GDR_ERR_WORKSPACE, "workspace of %zu bytes required (got %zu at %p)", need, workspace_bytes,
                    workspace);
    for (size_t i = 0; i < sizeof(outs) / sizeof(outs[0]); ++i) {
        for (const Span& s : ins)
            if (overlap(outs[i].p, outs[i].n, s.p, s.n))
                return fail(GDR_ERR_INVALID_ARG, "%s overlaps input %s", outs[i].name, s.name);
        for (size_t j = i + 1; j < sizeof(outs) / sizeof(outs[0]); ++j)
            if (overlap(outs[i].p, outs[i].n, outs[j].p, outs[j].n))
                return fail(GDR_ERR_INVALID_ARG, "%s overlaps %s", outs[i].name, outs[j].name);
        if (overlap(workspace, need, outs[i].p, outs[i].n))
            return fail(GDR_ERR_INVALID_ARG, "workspace overlaps %s", outs[i].name);
    }
    for (const Span& s : ins)
        if (overlap(workspace, need, s.p, s.n)) return fail(GDR_ERR_INVALID_ARG, "workspace overlaps %s", s.name);
    int* status = nullptr;
    int major = 0;
    if (int rc = device_setup(&status, &major)) return rc;
    if (major != 10) return fail(GDR_ERR_DEVICE, "compute capability %d.x: this library is built for sm_100a", major);
    BwdProblem p{q, k, v, g, beta, S0, dO, dS_T, dq, dk_out, dv_out, dg, dbeta, dS0, workspace,
                 B, T, H, dk, dv, mode, dtype, (float)(1.0 / sqrt((double)dk)), status};
    const cudaError_t err = launch_bwd(p, static_cast<cudaStream_t>(stream));
    if (err != cudaSuccess) return fail(GDR_ERR_CUDA, "backward launch: %s", cudaGetErrorString(err));
    return ok();
}

int gdr_sync_status(void* stream) {
    int* status = nullptr;
    int major = 0;
    if (int rc = device_setup(&status, &major)) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t err = cudaStreamSynchronize(s);
    if (err != cudaSuccess) return fail(GDR_ERR_CUDA, "stream error: %s", cudaGetErrorString(err));
    int rec[kStatusWords] = {};
    err = cudaMemcpyAsync(rec, status, sizeof(rec), cudaMemcpyDeviceToHost, s);
    if (err == cudaSuccess) err = cudaMemsetAsync(status, 0, sizeof(rec), s);
    if (err == cudaSuccess) err = cudaStreamSynchronize(s);
    if (err != cudaSuccess) return fail(GDR_ERR_CUDA, "reading the status word: %s", cudaGetErrorString(err));
    const int h = rec[0];
    if (h == GDR_ERR_TIMEOUT)
        return fail(GDR_ERR_TIMEOUT,
                    "a kernel's bounded wait expired; its outputs are invalid (wait kind %d, block %d, thread %d, "
                    "detail 0x%08x)",
                    rec[1], rec[2], rec[3], (unsigned)rec[4]);
    if (h == GDR_ERR_RANGE)
        return fail(GDR_ERR_RANGE, "a value left the range a kernel supports");
    if (h != 0) return fail(h, "device reported status %d", h);
    return ok();
}

int gdr_selftest_bounded_wait(unsigned limit_us, unsigned long long* elapsed_ns, void* stream) {
    if (limit_us == 0 || limit_us > 1000000u)
        return fail(GDR_ERR_INVALID_ARG, "limit_us = %u (1 .. 1000000)", limit_us);
    int* status = nullptr;
    int major = 0;
    if (int rc = device_setup(&status, &major)) return rc;
    if (major != 10) return fail(GDR_ERR_DEVICE, "compute capability %d.x: this library is built for sm_100a", major);
    const int before = gdr_sync_status(stream);  // an idle stream and a clear status word to start from
    if (before == GDR_ERR_CUDA) return before;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const cudaError_t err = launch_bounded_wait_selftest(status, (uint64_t)limit_us * 1000ull, s);
    if (err != cudaSuccess) return fail(GDR_ERR_CUDA, "self-test launch: %s", cudaGetErrorString(err));
    const int rc = gdr_sync_status(stream);
    if (elapsed_ns != nullptr && read_bounded_wait_selftest_elapsed(elapsed_ns) != cudaSuccess) *elapsed_ns = 0;
    return rc;
}

}  // extern "C"

// ----------------------------------------------------------- allocation-free variant --
// gdr_chunk_fwd_noalloc: the tensor-core chunked forward for callers that cannot allocate device
// memory (see include/gdr.h for who they are). Its scratch is this fixed area, part of the
// library's device image: every GPU that loads the library holds it until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[GDR_NOALLOC_SCRATCH_BYTES];

namespace gdr {
namespace {

void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch area on the current device. In host code the array's name is
// only a host-side stand-in, so the address is looked up once per device, with it current.
int noalloc_scratch(void** ptr) {
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return fail(GDR_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(err));
    if (dev < 0 || dev >= kMaxDevices) return fail(GDR_ERR_DEVICE, "device ordinal %d out of range", dev);
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    if (g_noalloc_ptr[dev] == nullptr) {
        void* p = nullptr;
        err = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (err != cudaSuccess)
            return fail(GDR_ERR_CUDA, "cudaGetSymbolAddress(scratch area): %s", cudaGetErrorString(err));
        g_noalloc_ptr[dev] = p;
    }
    *ptr = g_noalloc_ptr[dev];
    return GDR_OK;
}

}  // namespace
}  // namespace gdr

extern "C" int gdr_chunk_fwd_noalloc(const void* q, const void* k, const void* v, const float* g, const float* beta,
                                     const float* S0, void* o, float* S_T, int B, int T, int H, int dk, int dv,
                                     int chunk, int mode, int dtype, int o_dtype, void* stream) {
    ProfileScope prof_scope;
    if (int rc = chunk_shape_check(B, T, H, dk, dv, chunk, mode, dtype, o_dtype)) return rc;
    if (!chunk_tc_supported(dk, dv, chunk, dtype, o_dtype))
        return fail(GDR_ERR_UNSUPPORTED,
                    "gdr_chunk_fwd_noalloc covers the shapes that need scratch (bf16 q/k/v, d_k = d_v = 128, "
                    "chunk 64); this shape needs none: call gdr_chunk_fwd with a null workspace");
    const size_t need = chunk_tc_workspace_bytes(B, T, H, dk, dv, chunk, mode);
    if (need > (size_t)GDR_NOALLOC_SCRATCH_BYTES)
        return fail(GDR_ERR_UNSUPPORTED,
                    "this problem needs %zu bytes of scratch but the built-in area holds %zu; "
                    "use gdr_chunk_fwd with a workspace",
                    need, (size_t)GDR_NOALLOC_SCRATCH_BYTES);
    void* ws = nullptr;
    if (int rc = noalloc_scratch(&ws)) return rc;
    return chunk_fwd_impl(q, k, v, g, beta, S0, o, S_T, B, T, H, dk, dv, chunk, mode, dtype, o_dtype, GDR_PRO_NONE,
                          nullptr, -1, nullptr, nullptr, ws, (size_t)GDR_NOALLOC_SCRATCH_BYTES, stream);
}

// ------------------------------------------------------------ host-buffer entry point --
namespace gdr {
namespace {

constexpr int kHostMaxPieces = 8;

size_t align256(size_t n) { return (n + 255) & ~size_t(255); }

// Byte sizes of the per-sequence slices of each tensor.
struct SeqBytes {
    size_t q, v, g, beta, s, o;
};
SeqBytes seq_bytes(int T, int H, int dk, int dv, int mode, int dtype, int o_dtype) {
    const size_t ntok = (size_t)T * H, eb = elem_bytes(dtype);
    SeqBytes r;
    r.q = ntok * dk * eb;
    r.v = ntok * dv * eb;
    r.g = mode == GDR_DECAY_NONE ? 0 : (mode == GDR_DECAY_SCALAR ? ntok * sizeof(float) : ntok * dk * sizeof(float));
    r.beta = ntok * sizeof(float);
    r.s = (size_t)H * dv * dk * sizeof(float);
    r.o = ntok * dv * elem_bytes(o_dtype);
    return r;
}

// Sequences per piece and the bytes of one staging slot (inputs, outputs and workspace of a piece).
void host_plan(int B, int T, int H, int dk, int dv, int chunk, int mode, int dtype, int o_dtype, int* pb,
               size_t* slot) {
    const int pieces = B < kHostMaxPieces ? B : kHostMaxPieces;
    *pb = (B + pieces - 1) / pieces;
    const SeqBytes sb = seq_bytes(T, H, dk, dv, mode, dtype, o_dtype);
    const size_t n = (size_t)*pb;
    const size_t ws = chunk_tc_supported(dk, dv, chunk, dtype, o_dtype)
                          ? chunk_tc_workspace_bytes(*pb, T, H, dk, dv, chunk, mode)
                          : 0;
    *slot = 3 * align256(n * sb.q) + align256(n * sb.g) + align256(n * sb.beta) + 2 * align256(n * sb.s) +
            align256(n * sb.o) + align256(ws);
}

struct HostStreams {
    cudaStream_t h2d = nullptr, d2h = nullptr;
    cudaEvent_t start = nullptr, in_ready[2] = {}, computed[2] = {}, out_done[2] = {};
};
HostStreams g_host[kMaxDevices];
// Held by a gdr_chunk_fwd_host call while it enqueues: the copy streams and events above are
// shared by every call on the device, so two threads must not interleave their records and waits.
std::mutex g_host_enqueue[kMaxDevices];

int host_streams(HostStreams** out, int* device) {
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return fail(GDR_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(err));
    if (dev < 0 || dev >= kMaxDevices) return fail(GDR_ERR_DEVICE, "device ordinal %d out of range", dev);
    *device = dev;
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    HostStreams& hs = g_host[dev];
    if (hs.h2d == nullptr) {
        HostStreams t;
        const unsigned ef = cudaEventDisableTiming;
        err = cudaStreamCreateWithFlags(&t.h2d, cudaStreamNonBlocking);
        if (err == cudaSuccess) err = cudaStreamCreateWithFlags(&t.d2h, cudaStreamNonBlocking);
        if (err == cudaSuccess) err = cudaEventCreateWithFlags(&t.start, ef);
        for (int i = 0; i < 2 && err == cudaSuccess; ++i) {
            err = cudaEventCreateWithFlags(&t.in_ready[i], ef);
            if (err == cudaSuccess) err = cudaEventCreateWithFlags(&t.computed[i], ef);
            if (err == cudaSuccess) err = cudaEventCreateWithFlags(&t.out_done[i], ef);
        }
        if (err != cudaSuccess) return fail(GDR_ERR_CUDA, "copy streams: %s", cudaGetErrorString(err));
        hs = t;
    }
    *out = &hs;
    return GDR_OK;
}

}  // namespace
}  // namespace gdr

extern "C" size_t gdr_chunk_fwd_host_staging_bytes(int B, int T, int H, int dk, int dv, int chunk, int mode,
                                                   int dtype, int o_dtype) {
    char saved[sizeof(g_last_error)];
    memcpy(saved, g_last_error, sizeof(saved));
    const int rc = chunk_shape_check(B, T, H, dk, dv, chunk, mode, dtype, o_dtype);
    memcpy(g_last_error, saved, sizeof(saved));
    if (rc != GDR_OK) return 0;
    int pb = 0;
    size_t slot = 0;
    host_plan(B, T, H, dk, dv, chunk, mode, dtype, o_dtype, &pb, &slot);
    return 2 * slot;
}

extern "C" int gdr_chunk_fwd_host(const void* q, const void* k, const void* v, const float* g, const float* beta,
                                  const float* S0, void* o, float* S_T, int B, int T, int H, int dk, int dv,
                                  int chunk, int mode, int dtype, int o_dtype, void* staging, size_t staging_bytes,
                                  void* stream) {
    ProfileScope prof_scope;
    if (int rc = chunk_shape_check(B, T, H, dk, dv, chunk, mode, dtype, o_dtype)) return rc;
    if (!q || !k || !v || !beta || !o) return fail(GDR_ERR_INVALID_ARG, "q, k, v, beta and o must be non-null");
    if (mode != GDR_DECAY_NONE && !g) return fail(GDR_ERR_INVALID_ARG, "g must be non-null for a gated decay mode");
    int pb = 0;
    size_t slot = 0;
    host_plan(B, T, H, dk, dv, chunk, mode, dtype, o_dtype, &pb, &slot);
    if (staging == nullptr || staging_bytes < 2 * slot)
        return fail(GDR_ERR_WORKSPACE, "staging of %zu bytes required (got %zu at %p)", 2 * slot, staging_bytes,
                    staging);
    if (!aligned16(staging)) return fail(GDR_ERR_MISALIGNED, "staging %p is not 16-byte aligned", staging);
    int* status = nullptr;
    int major = 0;
    if (int rc = device_setup(&status, &major)) return rc;
    if (major != 10) return fail(GDR_ERR_DEVICE, "compute capability %d.x: this library is built for sm_100a", major);
    HostStreams* hs = nullptr;
    int hdev = 0;
    if (int rc = host_streams(&hs, &hdev)) return rc;
    // the whole enqueue sequence below uses the device's shared copy streams and events
    std::lock_guard<std::mutex> enqueue_lock(g_host_enqueue[hdev]);

    const SeqBytes sb = seq_bytes(T, H, dk, dv, mode, dtype, o_dtype);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    auto cuda_fail = [&](cudaError_t e, const char* what) {
        return fail(GDR_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    };
    cudaError_t err = cudaEventRecord(hs->start, s);  // everything below follows the work already on `stream`
    if (err != cudaSuccess) return cuda_fail(err, "event record");
    if ((err = cudaStreamWaitEvent(hs->h2d, hs->start, 0)) != cudaSuccess) return cuda_fail(err, "stream wait");
    const size_t sz = (size_t)pb;
    int piece = 0;
    for (int b0 = 0; b0 < B; b0 += pb, ++piece) {
        const int nb = B - b0 < pb ? B - b0 : pb;
        const int sl = piece & 1;
        uint8_t* base = static_cast<uint8_t*>(staging) + sl * slot;
        uint8_t* dq = base;
        uint8_t* dk_ = dq + align256(sz * sb.q);
        uint8_t* dv_ = dk_ + align256(sz * sb.q);
        uint8_t* dg = dv_ + align256(sz * sb.v);
        uint8_t* dbeta = dg + align256(sz * sb.g);
        uint8_t* ds0 = dbeta + align256(sz * sb.beta);
        uint8_t* dst = ds0 + align256(sz * sb.s);
        uint8_t* dout = dst + align256(sz * sb.s);
        uint8_t* dws = dout + align256(sz * sb.o);
        const size_t ws_bytes = slot - (size_t)(dws - base);
        // inputs of this piece (after the outputs of the piece that used this slot two steps ago)
        if (piece >= 2 && (err = cudaStreamWaitEvent(hs->h2d, hs->out_done[sl], 0)) != cudaSuccess)
            return cuda_fail(err, "stream wait");
        struct Cp { void* d; const void* h; size_t n; };
        const Cp in[] = {{dq, static_cast<const uint8_t*>(q) + b0 * sb.q, nb * sb.q},
                         {dk_, static_cast<const uint8_t*>(k) + b0 * sb.q, nb * sb.q},
                         {dv_, static_cast<const uint8_t*>(v) + b0 * sb.v, nb * sb.v},
                         {dg, g ? reinterpret_cast<const uint8_t*>(g) + b0 * sb.g : nullptr, nb * sb.g},
                         {dbeta, reinterpret_cast<const uint8_t*>(beta) + b0 * sb.beta, nb * sb.beta},
                         {ds0, S0 ? reinterpret_cast<const uint8_t*>(S0) + b0 * sb.s : nullptr, nb * sb.s}};
        for (const Cp& c : in)
            if (c.h != nullptr && c.n > 0 &&
                (err = cudaMemcpyAsync(c.d, c.h, c.n, cudaMemcpyHostToDevice, hs->h2d)) != cudaSuccess)
                return cuda_fail(err, "copy in");
        if ((err = cudaEventRecord(hs->in_ready[sl], hs->h2d)) != cudaSuccess) return cuda_fail(err, "event record");
        // the piece's forward on `stream`
        if ((err = cudaStreamWaitEvent(s, hs->in_ready[sl], 0)) != cudaSuccess) return cuda_fail(err, "stream wait");
        const int rc = gdr_chunk_fwd(dq, dk_, dv_, g ? reinterpret_cast<const float*>(dg) : nullptr,
                                     reinterpret_cast<const float*>(dbeta), S0 ? reinterpret_cast<const float*>(ds0) : nullptr,
                                     dout, S_T ? reinterpret_cast<float*>(dst) : nullptr, nb, T, H, dk, dv, chunk, mode,
                                     dtype, o_dtype, dws, ws_bytes, s);
        if (rc != GDR_OK) return rc;
        if ((err = cudaEventRecord(hs->computed[sl], s)) != cudaSuccess) return cuda_fail(err, "event record");
        // outputs of this piece
        if ((err = cudaStreamWaitEvent(hs->d2h, hs->computed[sl], 0)) != cudaSuccess) return cuda_fail(err, "stream wait");
        if ((err = cudaMemcpyAsync(static_cast<uint8_t*>(o) + b0 * sb.o, dout, nb * sb.o, cudaMemcpyDeviceToHost,
                                   hs->d2h)) != cudaSuccess)
            return cuda_fail(err, "copy out");
        if (S_T != nullptr &&
            (err = cudaMemcpyAsync(reinterpret_cast<uint8_t*>(S_T) + b0 * sb.s, dst, nb * sb.s, cudaMemcpyDeviceToHost,
                                   hs->d2h)) != cudaSuccess)
            return cuda_fail(err, "copy out");
        if ((err = cudaEventRecord(hs->out_done[sl], hs->d2h)) != cudaSuccess) return cuda_fail(err, "event record");
    }
    // `stream` completes after the last copy out (the copy-out stream runs the pieces in order)
    if ((err = cudaStreamWaitEvent(s, hs->out_done[(piece - 1) & 1], 0)) != cudaSuccess) return cuda_fail(err, "stream wait");
    return ok();
}
