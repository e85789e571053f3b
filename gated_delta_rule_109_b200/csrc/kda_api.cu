// libkda C ABI: argument validation, dispatch to the kernels, status codes.
// The contract of every entry point is documented in include/kda.h.
#include <algorithm>
#include <atomic>
#include <math.h>
#include <mutex>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "kda_internal.cuh"

namespace {

thread_local char g_last_cuda_error[256] = "";
std::atomic<unsigned long long> g_launches{0};

kda_status cuda_fail(cudaError_t e)
{
    snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "%s: %s",
             cudaGetErrorName(e), cudaGetErrorString(e));
    return KDA_ERR_CUDA;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
bool head_dim_ok(int d) { return d == 64 || d == 128; }

// Scratch of kda_forward_noalloc: part of the library's device image, so a call
// allocates nothing.  Its address is looked up once per device; an event per
// device orders the calls that use it, whatever their streams.
constexpr size_t kScratchBytes = size_t(128) << 20;
static __device__ __align__(256) uint8_t g_kda_scratch[kScratchBytes];
constexpr int kMaxDevices = 64;
struct ScratchSlot {
    void *ptr = nullptr;
    cudaEvent_t done = nullptr;
};
ScratchSlot g_scratch[kMaxDevices];
std::mutex g_scratch_mu;

// Workspace of kda_forward and kda_gdn_forward: one stream-ordered memory pool per
// device, owned by the library.  A call takes its workspace from the pool on its
// stream and gives it back on the same stream once its kernels are enqueued; the
// pool keeps up to kPoolKeep bytes between calls, so that after the first call of
// a shape the allocation is a lookup.  A call asks for at most kPoolKeep bytes
// unless the smallest workspace of its shape is larger.
constexpr size_t kPoolKeep = size_t(1) << 30;
cudaMemPool_t g_pool[kMaxDevices] = {};
std::mutex g_pool_mu;

cudaError_t device_pool(bool create, cudaMemPool_t *out)
{
    *out = nullptr;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_pool_mu);
    if (!g_pool[dev] && create) {
        cudaMemPoolProps props;
        memset(&props, 0, sizeof(props));
        props.allocType = cudaMemAllocationTypePinned;
        props.handleTypes = cudaMemHandleTypeNone;
        props.location.type = cudaMemLocationTypeDevice;
        props.location.id = dev;
        cudaMemPool_t pool = nullptr;
        if ((e = cudaMemPoolCreate(&pool, &props)) != cudaSuccess) return e;
        uint64_t keep = kPoolKeep;
        if ((e = cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep)) != cudaSuccess) {
            cudaMemPoolDestroy(pool);
            return e;
        }
        g_pool[dev] = pool;
    }
    *out = g_pool[dev];
    return cudaSuccess;
}

}  // namespace

void kda::note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

extern "C" {

unsigned long long kda_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }


int kda_version(void) { return 300; }   // 0.3.0

const char *kda_status_string(kda_status s)
{
    switch (s) {
    case KDA_OK: return "KDA_OK";
    case KDA_ERR_INVALID_ARG: return "KDA_ERR_INVALID_ARG";
    case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED";
    case KDA_ERR_MISALIGNED: return "KDA_ERR_MISALIGNED";
    case KDA_ERR_CUDA: return "KDA_ERR_CUDA";
    case KDA_ERR_TIMEOUT: return "KDA_ERR_TIMEOUT";
    }
    return "KDA_ERR_UNKNOWN";
}

const char *kda_last_cuda_error(void) { return g_last_cuda_error; }

}  // extern "C"

namespace {

// Argument checks of the forward entry points (nothing is enqueued unless all pass).
kda_status validate_forward(const void *q, const void *k, const void *v, const float *log_alpha,
                            const float *beta, const float *initial_state, float *out, float *final_state,
                            int B, int T, int H, int dk, int dv, kda_dtype dtype, float scale,
                            kda::GateKind gate, void *workspace)
{
    if (B <= 0 || H <= 0 || T < 0 || dk <= 0 || dv <= 0) return KDA_ERR_INVALID_ARG;
    if (dtype != KDA_BF16 && dtype != KDA_F32) return KDA_ERR_INVALID_ARG;
    if (!isfinite(scale)) return KDA_ERR_INVALID_ARG;
    if ((int64_t)B * H > (int64_t)INT32_MAX / 4) return KDA_ERR_INVALID_ARG;
    const bool need_gate = gate != kda::KDA_GATE_NONE;
    if (T > 0 && (!q || !k || !v || (need_gate && !log_alpha) || !beta || !out)) return KDA_ERR_INVALID_ARG;
    if (!head_dim_ok(dk) || !head_dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
    const bool gate_aligned = gate == kda::KDA_GATE_CHANNEL ? aligned16(log_alpha)
                              : gate == kda::KDA_GATE_SCALAR ? aligned4(log_alpha) : true;
    if (T > 0 && (!aligned16(q) || !aligned16(k) || !aligned16(v) || !gate_aligned ||
                  !aligned16(out) || !aligned4(beta)))
        return KDA_ERR_MISALIGNED;
    if ((initial_state && !aligned16(initial_state)) || (final_state && !aligned16(final_state)))
        return KDA_ERR_MISALIGNED;
    if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u)) return KDA_ERR_MISALIGNED;
    return KDA_OK;
}

// Shared by the per-channel (KDA) and scalar-gate (Gated DeltaNet / DeltaNet)
// entry points: they differ only in the shape of log_alpha.
kda_status forward_impl(const void *q, const void *k, const void *v, const float *log_alpha,
                        const float *beta, const float *initial_state, float *out, float *final_state,
                        int B, int T, int H, int dk, int dv, kda_dtype dtype, float scale,
                        void *stream, kda::GateKind gate, void *workspace = nullptr,
                        size_t workspace_bytes = 0, int prep_flags = 0, int T_whole = 0)
{
    g_last_cuda_error[0] = '\0';
    const kda_status vs = validate_forward(q, k, v, log_alpha, beta, initial_state, out, final_state, B, T, H,
                                           dk, dv, dtype, scale, gate, workspace);
    if (vs != KDA_OK) return vs;
    const bool need_gate = gate != kda::KDA_GATE_NONE;

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t state_bytes = sizeof(float) * (size_t)B * H * dk * dv;
    if (T == 0) {
        // no tokens: the final state is the initial state (or zeros)
        if (!final_state || final_state == initial_state) return KDA_OK;
        cudaError_t e = initial_state
            ? cudaMemcpyAsync(final_state, initial_state, state_bytes, cudaMemcpyDeviceToDevice, st)
            : cudaMemsetAsync(final_state, 0, state_bytes, st);
        return e == cudaSuccess ? KDA_OK : cuda_fail(e);
    }

    kda::ForwardArgs a;
    a.q = q; a.k = k; a.v = v; a.log_alpha = need_gate ? log_alpha : nullptr; a.beta = beta;
    a.s0 = initial_state; a.out = out; a.sT = final_state;
    a.B = B; a.T = T; a.H = H; a.dk = dk; a.dv = dv; a.dtype = dtype;
    a.scale = (scale == 0.0f) ? 1.0f / sqrtf((float)dk) : scale;
    a.gate = gate;
    a.prep_flags = prep_flags;
    cudaError_t e;
    if (workspace && kda::prefill_split_supported(a) &&
        workspace_bytes >= kda::prefill_split_workspace_min(B, T, H))
        e = kda::launch_prefill_split(a, static_cast<uint8_t *>(workspace), workspace_bytes, st, T_whole);
    else if (!kda::prefill_tc_supported(a)) e = kda::launch_prefill_simt(a, st);
    else if (gate == kda::KDA_GATE_CHANNEL) e = kda::launch_prefill_tc(a, st);
    else e = kda::launch_prefill_gdn_tc(a, st);
    return e == cudaSuccess ? KDA_OK : cuda_fail(e);
}

// kda_forward / kda_gdn_forward: the two-kernel prefill on a workspace from the
// library's pool where it applies (bf16, dk = dv = 128); the one-kernel prefill,
// which needs no memory beyond its arguments, for other shapes or when the pool
// cannot supply the workspace.
kda_status forward_pooled(const void *q, const void *k, const void *v, const float *log_alpha,
                          const float *beta, const float *initial_state, float *out, float *final_state,
                          int B, int T, int H, int dk, int dv, kda_dtype dtype, float scale,
                          void *stream, kda::GateKind gate)
{
    g_last_cuda_error[0] = '\0';
    const kda_status vs = validate_forward(q, k, v, log_alpha, beta, initial_state, out, final_state, B, T, H,
                                           dk, dv, dtype, scale, gate, nullptr);
    if (vs != KDA_OK) return vs;
    if (T == 0 || dtype != KDA_BF16 || dk != 128 || dv != 128)
        return forward_impl(q, k, v, log_alpha, beta, initial_state, out, final_state, B, T, H, dk, dv, dtype,
                            scale, stream, gate);
    const size_t want = std::max(std::min(kda::prefill_split_workspace_best(B, T, H), kPoolKeep),
                                 kda::prefill_split_workspace_min(B, T, H));
    cudaMemPool_t pool = nullptr;
    cudaError_t e = device_pool(true, &pool);
    if (e != cudaSuccess) return cuda_fail(e);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    void *ws = nullptr;
    if (cudaMallocFromPoolAsync(&ws, want, pool, st) != cudaSuccess) {
        cudaGetLastError();             // no room for the workspace: the one-kernel prefill
        return forward_impl(q, k, v, log_alpha, beta, initial_state, out, final_state, B, T, H, dk, dv, dtype,
                            scale, stream, gate);
    }
    const kda_status rs = forward_impl(q, k, v, log_alpha, beta, initial_state, out, final_state, B, T, H, dk,
                                       dv, dtype, scale, stream, gate, ws, want);
    e = cudaFreeAsync(ws, st);          // after every kernel of the call (they join the caller's stream)
    if (rs != KDA_OK) return rs;
    return e == cudaSuccess ? KDA_OK : cuda_fail(e);
}

kda_status decode_impl(const void *q, const void *k, const void *v, const float *log_alpha,
                       const float *beta, float *state_inout, float *out, int B, int H, int dk, int dv,
                       kda_dtype dtype, float scale, void *stream, kda::GateKind gate)
{
    g_last_cuda_error[0] = '\0';
    if (B <= 0 || H <= 0 || dk <= 0 || dv <= 0) return KDA_ERR_INVALID_ARG;
    if (dtype != KDA_BF16 && dtype != KDA_F32) return KDA_ERR_INVALID_ARG;
    if (!isfinite(scale)) return KDA_ERR_INVALID_ARG;
    // the decode grid has up to 4 CTAs per head (two per 128 value columns, with
    // room for one more split); keep B * H * 4 within a grid dimension
    if ((int64_t)B * H > (int64_t)INT32_MAX / 4) return KDA_ERR_INVALID_ARG;
    const bool need_gate = gate != kda::KDA_GATE_NONE;
    if (!q || !k || !v || (need_gate && !log_alpha) || !beta || !state_inout || !out)
        return KDA_ERR_INVALID_ARG;
    if (!head_dim_ok(dk) || !head_dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
    const bool gate_aligned = gate == kda::KDA_GATE_CHANNEL ? aligned16(log_alpha)
                              : gate == kda::KDA_GATE_SCALAR ? aligned4(log_alpha) : true;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !gate_aligned ||
        !aligned16(state_inout) || !aligned16(out) || !aligned4(beta))
        return KDA_ERR_MISALIGNED;

    kda::DecodeArgs a;
    a.q = q; a.k = k; a.v = v; a.log_alpha = need_gate ? log_alpha : nullptr; a.beta = beta;
    a.state = state_inout; a.out = out;
    a.B = B; a.H = H; a.dk = dk; a.dv = dv; a.dtype = dtype;
    a.scale = (scale == 0.0f) ? 1.0f / sqrtf((float)dk) : scale;
    a.gate = gate;
    cudaError_t e = kda::launch_decode(a, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? KDA_OK : cuda_fail(e);
}

// kda_forward_host: per-device copy streams and the events that order the slots
struct HostPipe {
    bool ready = false;
    cudaStream_t h2d = nullptr, d2h = nullptr;
    cudaEvent_t in_ready[2], comp_done[2], out_done[2], start, fin;
};
HostPipe g_pipe[kMaxDevices];
std::mutex g_pipe_mu;

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

// Workspace of kda_forward_host: two input slots and two output slots of one block
// of tokens each, the carried state, and the two-kernel records of one block.
struct HostLayout {
    int Tb;
    size_t q, k, v, la, beta, slot_in, slot_out, state, recs, recs_bytes, total;
};
HostLayout host_layout(int B, int T, int H, int dk, int dv, kda_dtype dtype, int block_tokens)
{
    HostLayout L;
    const int want = block_tokens > 0 ? ((block_tokens + 63) / 64) * 64 : 8192;
    L.Tb = (int)std::min<long long>(want, ((long long)T + 63) / 64 * 64);
    if (L.Tb <= 0) L.Tb = 64;
    const size_t esz = dtype == KDA_BF16 ? 2 : 4, rows = (size_t)B * L.Tb * H;
    L.q = 0;
    L.k = L.q + up256(rows * dk * esz);
    L.v = L.k + up256(rows * dk * esz);
    L.la = L.v + up256(rows * dv * esz);
    L.beta = L.la + up256(rows * dk * 4);
    L.slot_in = L.beta + up256(rows * 4);
    L.slot_out = up256(rows * dv * 4);
    L.state = 2 * L.slot_in + 2 * L.slot_out;
    L.recs = L.state + up256((size_t)B * H * dk * dv * 4);
    L.recs_bytes = (dtype == KDA_BF16 && dk == 128 && dv == 128) ? kda::prefill_split_workspace_full(B, L.Tb, H) : 0;
    L.total = L.recs + L.recs_bytes;
    return L;
}

}  // namespace

extern "C" {

kda_status kda_forward(const void *q, const void *k, const void *v,
                       const float *log_alpha, const float *beta,
                       const float *initial_state, float *out, float *final_state,
                       int B, int T, int H, int dk, int dv,
                       kda_dtype dtype, float scale, void *stream)
{
    return forward_pooled(q, k, v, log_alpha, beta, initial_state, out, final_state, B, T, H, dk, dv,
                          dtype, scale, stream, kda::KDA_GATE_CHANNEL);
}

kda_status kda_forward_raw(const void *q, const void *k, const void *v,
                           const float *gate, const float *beta,
                           const float *initial_state, float *out, float *final_state,
                           int B, int T, int H, int dk, int dv,
                           kda_dtype dtype, float scale, unsigned int prep,
                           void *workspace, size_t workspace_bytes, void *stream)
{
    g_last_cuda_error[0] = '\0';
    if (prep & ~(unsigned)(KDA_PREP_LOGSIGMOID_GATE | KDA_PREP_L2NORM_QK)) return KDA_ERR_INVALID_ARG;
    const kda_status vs = validate_forward(q, k, v, gate, beta, initial_state, out, final_state, B, T, H, dk, dv,
                                           dtype, scale, kda::KDA_GATE_CHANNEL, workspace);
    if (vs != KDA_OK) return vs;
    if (prep != 0 && T > 0) {
        // the fused steps live in the two-kernel prefill's first kernel
        if (dtype != KDA_BF16 || dk != 128 || dv != 128 || !workspace ||
            workspace_bytes < kda::prefill_split_workspace_min(B, T, H))
            return KDA_ERR_UNSUPPORTED;
    }
    return forward_impl(q, k, v, gate, beta, initial_state, out, final_state, B, T, H, dk, dv, dtype, scale,
                        stream, kda::KDA_GATE_CHANNEL, workspace, workspace_bytes, (int)prep);
}

kda_status kda_segment_local(const void *q, const void *k, const void *v,
                             const float *log_alpha, const float *beta,
                             const float *initial_state, float *out, float *local_final, float *transfer,
                             int B, int T, int H, int dk, int dv,
                             kda_dtype dtype, float scale, void *workspace, size_t workspace_bytes, void *stream)
{
    g_last_cuda_error[0] = '\0';
    if (T <= 0 || !local_final || !transfer) return KDA_ERR_INVALID_ARG;
    const kda_status vs = validate_forward(q, k, v, log_alpha, beta, initial_state, out, local_final, B, T, H, dk,
                                           dv, dtype, scale, kda::KDA_GATE_CHANNEL, workspace);
    if (vs != KDA_OK) return vs;
    if (!aligned16(transfer)) return KDA_ERR_MISALIGNED;
    if (dtype != KDA_BF16 || dk != 128 || dv != 128 || !workspace ||
        workspace_bytes < kda::prefill_split_workspace_full(B, T, H))
        return KDA_ERR_UNSUPPORTED;
    kda::ForwardArgs a;
    a.q = q; a.k = k; a.v = v; a.log_alpha = log_alpha; a.beta = beta;
    a.s0 = initial_state; a.out = out; a.sT = local_final;
    a.B = B; a.T = T; a.H = H; a.dk = dk; a.dv = dv; a.dtype = dtype;
    a.scale = (scale == 0.0f) ? 1.0f / sqrtf((float)dk) : scale;
    a.gate = kda::KDA_GATE_CHANNEL;
    a.prep_flags = 0;
    const cudaError_t e = kda::launch_segment_local(a, transfer, static_cast<uint8_t *>(workspace),
                                                    static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? KDA_OK : cuda_fail(e);
}

kda_status kda_segment_start_state(const float *transfers, const float *local_finals, int R,
                                   float *start, int B, int H, int dk, int dv, void *stream)
{
    g_last_cuda_error[0] = '\0';
    if (R < 1 || B <= 0 || H <= 0 || !transfers || !local_finals || !start) return KDA_ERR_INVALID_ARG;
    if ((int64_t)B * H > (int64_t)INT32_MAX / 4) return KDA_ERR_INVALID_ARG;
    if (dk != 128 || dv != 128) return KDA_ERR_UNSUPPORTED;
    if (!aligned16(transfers) || !aligned16(local_finals) || !aligned16(start)) return KDA_ERR_MISALIGNED;
    const cudaError_t e = kda::launch_affine_compose(transfers, local_finals, R, B * H, start,
                                                     static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? KDA_OK : cuda_fail(e);
}

kda_status kda_segment_correct(const float *start, const float *local_final, float *out, float *final_state,
                               int B, int T, int H, int dk, int dv,
                               const void *workspace, size_t workspace_bytes, void *stream)
{
    g_last_cuda_error[0] = '\0';
    if (B <= 0 || H <= 0 || T <= 0 || !start || !local_final || !out || !workspace) return KDA_ERR_INVALID_ARG;
    if ((int64_t)B * H > (int64_t)INT32_MAX / 4) return KDA_ERR_INVALID_ARG;
    if (dk != 128 || dv != 128) return KDA_ERR_UNSUPPORTED;
    if (!aligned16(start) || !aligned16(local_final) || !aligned16(out) ||
        (final_state && !aligned16(final_state)) || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return KDA_ERR_MISALIGNED;
    if (workspace_bytes < kda::prefill_split_workspace_full(B, T, H)) return KDA_ERR_UNSUPPORTED;
    kda::ForwardArgs a = {};
    a.out = out; a.sT = final_state;
    a.B = B; a.T = T; a.H = H; a.dk = dk; a.dv = dv; a.dtype = KDA_BF16;
    a.gate = kda::KDA_GATE_CHANNEL;
    const cudaError_t e = kda::launch_segment_correct(a, start, local_final, static_cast<const uint8_t *>(workspace),
                                                      static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? KDA_OK : cuda_fail(e);
}

size_t kda_forward_workspace_bytes(int B, int T, int H, int dk, int dv, kda_dtype dtype)
{
    if (B <= 0 || H <= 0 || T <= 0 || dtype != KDA_BF16 || dk != 128 || dv != 128) return 0;
    return kda::prefill_split_workspace_best(B, T, H);
}

size_t kda_segment_workspace_bytes(int B, int T, int H, int dk, int dv, kda_dtype dtype)
{
    if (B <= 0 || H <= 0 || T <= 0 || dtype != KDA_BF16 || dk != 128 || dv != 128) return 0;
    return kda::prefill_split_workspace_full(B, T, H);
}

size_t kda_forward_workspace_min_bytes(int B, int T, int H, int dk, int dv, kda_dtype dtype)
{
    if (B <= 0 || H <= 0 || T <= 0 || dtype != KDA_BF16 || dk != 128 || dv != 128) return 0;
    return kda::prefill_split_workspace_min(B, T, H);
}

kda_status kda_forward_ws(const void *q, const void *k, const void *v,
                          const float *log_alpha, const float *beta,
                          const float *initial_state, float *out, float *final_state,
                          int B, int T, int H, int dk, int dv,
                          kda_dtype dtype, float scale, void *workspace, size_t workspace_bytes,
                          void *stream)
{
    return forward_impl(q, k, v, log_alpha, beta, initial_state, out, final_state, B, T, H, dk, dv,
                        dtype, scale, stream, kda::KDA_GATE_CHANNEL, workspace, workspace_bytes);
}

kda_status kda_forward_noalloc(const void *q, const void *k, const void *v,
                               const float *log_alpha, const float *beta,
                               const float *initial_state, float *out, float *final_state,
                               int B, int T, int H, int dk, int dv,
                               kda_dtype dtype, float scale, void *stream)
{
    g_last_cuda_error[0] = '\0';
    const kda_status vs = validate_forward(q, k, v, log_alpha, beta, initial_state, out, final_state, B, T, H,
                                           dk, dv, dtype, scale, kda::KDA_GATE_CHANNEL, nullptr);
    if (vs != KDA_OK) return vs;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (dev < 0 || dev >= kMaxDevices) return KDA_ERR_UNSUPPORTED;
    ScratchSlot &slot = g_scratch[dev];
    if (!slot.ptr) {
        void *ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, g_kda_scratch);
        if (e == cudaSuccess && !slot.done) e = cudaEventCreateWithFlags(&slot.done, cudaEventDisableTiming);
        if (e != cudaSuccess) return cuda_fail(e);
        slot.ptr = ptr;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    e = cudaStreamWaitEvent(st, slot.done, 0);          // the previous user of the scratch is done
    if (e != cudaSuccess) return cuda_fail(e);
    const kda_status rs = forward_impl(q, k, v, log_alpha, beta, initial_state, out, final_state, B, T, H, dk,
                                       dv, dtype, scale, stream, kda::KDA_GATE_CHANNEL, slot.ptr, kScratchBytes);
    e = cudaEventRecord(slot.done, st);
    if (rs != KDA_OK) return rs;
    return e == cudaSuccess ? KDA_OK : cuda_fail(e);
}

size_t kda_forward_noalloc_scratch_bytes(void) { return kScratchBytes; }

size_t kda_workspace_pool_bytes(void)
{
    cudaMemPool_t pool = nullptr;
    if (device_pool(false, &pool) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    uint64_t held = 0;
    if (!pool || cudaMemPoolGetAttribute(pool, cudaMemPoolAttrReservedMemCurrent, &held) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    return (size_t)held;
}

kda_status kda_workspace_pool_trim(void *stream)
{
    g_last_cuda_error[0] = '\0';
    cudaMemPool_t pool = nullptr;
    cudaError_t e = device_pool(false, &pool);
    if (e != cudaSuccess) return cuda_fail(e);
    if (!pool) return KDA_OK;
    // the calls already enqueued on the stream give their workspaces back first
    if ((e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream))) != cudaSuccess) return cuda_fail(e);
    e = cudaMemPoolTrimTo(pool, 0);
    return e == cudaSuccess ? KDA_OK : cuda_fail(e);
}

kda_status kda_decode_step(const void *q, const void *k, const void *v,
                           const float *log_alpha, const float *beta,
                           float *state_inout, float *out,
                           int B, int H, int dk, int dv,
                           kda_dtype dtype, float scale, void *stream)
{
    return decode_impl(q, k, v, log_alpha, beta, state_inout, out, B, H, dk, dv, dtype, scale, stream,
                       kda::KDA_GATE_CHANNEL);
}

kda_status kda_gdn_forward(const void *q, const void *k, const void *v,
                           const float *log_alpha, const float *beta,
                           const float *initial_state, float *out, float *final_state,
                           int B, int T, int H, int dk, int dv,
                           kda_dtype dtype, float scale, void *stream)
{
    return forward_pooled(q, k, v, log_alpha, beta, initial_state, out, final_state, B, T, H, dk, dv,
                          dtype, scale, stream, log_alpha ? kda::KDA_GATE_SCALAR : kda::KDA_GATE_NONE);
}

kda_status kda_gdn_forward_ws(const void *q, const void *k, const void *v,
                              const float *log_alpha, const float *beta,
                              const float *initial_state, float *out, float *final_state,
                              int B, int T, int H, int dk, int dv,
                              kda_dtype dtype, float scale, void *workspace, size_t workspace_bytes, void *stream)
{
    return forward_impl(q, k, v, log_alpha, beta, initial_state, out, final_state, B, T, H, dk, dv,
                        dtype, scale, stream, log_alpha ? kda::KDA_GATE_SCALAR : kda::KDA_GATE_NONE,
                        workspace, workspace_bytes);
}

kda_status kda_gdn_decode_step(const void *q, const void *k, const void *v,
                               const float *log_alpha, const float *beta,
                               float *state_inout, float *out,
                               int B, int H, int dk, int dv,
                               kda_dtype dtype, float scale, void *stream)
{
    return decode_impl(q, k, v, log_alpha, beta, state_inout, out, B, H, dk, dv, dtype, scale, stream,
                       log_alpha ? kda::KDA_GATE_SCALAR : kda::KDA_GATE_NONE);
}

size_t kda_forward_host_workspace_bytes(int B, int T, int H, int dk, int dv, kda_dtype dtype, int block_tokens)
{
    if (B <= 0 || H <= 0 || T < 0 || !head_dim_ok(dk) || !head_dim_ok(dv) || block_tokens < 0 ||
        (dtype != KDA_BF16 && dtype != KDA_F32))
        return 0;
    return host_layout(B, T, H, dk, dv, dtype, block_tokens).total;
}

kda_status kda_forward_host(const void *q, const void *k, const void *v,
                            const float *log_alpha, const float *beta,
                            const float *initial_state, float *out, float *final_state,
                            int B, int T, int H, int dk, int dv,
                            kda_dtype dtype, float scale, int block_tokens,
                            void *workspace, size_t workspace_bytes, void *stream)
{
    g_last_cuda_error[0] = '\0';
    if (B <= 0 || H <= 0 || T < 0 || dk <= 0 || dv <= 0 || block_tokens < 0) return KDA_ERR_INVALID_ARG;
    if (dtype != KDA_BF16 && dtype != KDA_F32) return KDA_ERR_INVALID_ARG;
    if (!isfinite(scale)) return KDA_ERR_INVALID_ARG;
    if (!head_dim_ok(dk) || !head_dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
    if ((int64_t)B * T * H > (int64_t)INT32_MAX / 4) return KDA_ERR_INVALID_ARG;
    const size_t esz = dtype == KDA_BF16 ? 2 : 4;
    const size_t state_bytes = sizeof(float) * (size_t)B * H * dk * dv;
    if (T == 0) {
        // no tokens: the final state is the initial state (or zeros), copied on the host
        if (final_state && final_state != initial_state) {
            if (initial_state) memcpy(final_state, initial_state, state_bytes);
            else memset(final_state, 0, state_bytes);
        }
        return KDA_OK;
    }
    if (!q || !k || !v || !log_alpha || !beta || !out || !workspace) return KDA_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return KDA_ERR_MISALIGNED;
    const HostLayout L = host_layout(B, T, H, dk, dv, dtype, block_tokens);
    if (workspace_bytes < L.total) return KDA_ERR_INVALID_ARG;

    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (dev < 0 || dev >= kMaxDevices) return KDA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_pipe_mu);
    HostPipe &P = g_pipe[dev];
    if (!P.ready) {
        if ((e = cudaStreamCreateWithFlags(&P.h2d, cudaStreamNonBlocking)) != cudaSuccess ||
            (e = cudaStreamCreateWithFlags(&P.d2h, cudaStreamNonBlocking)) != cudaSuccess)
            return cuda_fail(e);
        for (cudaEvent_t *ev : {&P.in_ready[0], &P.in_ready[1], &P.comp_done[0], &P.comp_done[1],
                                &P.out_done[0], &P.out_done[1], &P.start, &P.fin})
            if ((e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming)) != cudaSuccess) return cuda_fail(e);
        P.ready = true;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    float *carry = reinterpret_cast<float *>(ws + L.state);
    // the copies wait for the work already on the caller's stream (earlier users of the workspace)
    if ((e = cudaEventRecord(P.start, st)) != cudaSuccess || (e = cudaStreamWaitEvent(P.h2d, P.start, 0)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(P.d2h, P.start, 0)) != cudaSuccess)
        return cuda_fail(e);
    if (initial_state &&
        (e = cudaMemcpyAsync(carry, initial_state, state_bytes, cudaMemcpyHostToDevice, P.h2d)) != cudaSuccess)
        return cuda_fail(e);
    const int nblk = (T + L.Tb - 1) / L.Tb;
    const size_t HK = (size_t)H * dk, HV = (size_t)H * dv;
    for (int i = 0; i < nblk; ++i) {
        const int t0 = i * L.Tb, Ti = min(L.Tb, T - t0), sl = i & 1;
        uint8_t *in = ws + sl * L.slot_in;
        uint8_t *dq = in + L.q, *dk_ = in + L.k, *dvv = in + L.v;
        float *dla = reinterpret_cast<float *>(in + L.la), *dbt = reinterpret_cast<float *>(in + L.beta);
        float *dout = reinterpret_cast<float *>(ws + 2 * L.slot_in + sl * L.slot_out);
        // block i's inputs: the slot was last read by block i - 2's kernels
        if (i >= 2 && (e = cudaStreamWaitEvent(P.h2d, P.comp_done[sl], 0)) != cudaSuccess) return cuda_fail(e);
        for (int b = 0; b < B; ++b) {
            const size_t src_row = (size_t)b * T + t0, dst_row = (size_t)b * Ti;
            struct { void *dst; const void *src; size_t bytes; } cps[5] = {
                {dq + dst_row * HK * esz, static_cast<const uint8_t *>(q) + src_row * HK * esz, Ti * HK * esz},
                {dk_ + dst_row * HK * esz, static_cast<const uint8_t *>(k) + src_row * HK * esz, Ti * HK * esz},
                {dvv + dst_row * HV * esz, static_cast<const uint8_t *>(v) + src_row * HV * esz, Ti * HV * esz},
                {dla + dst_row * HK, log_alpha + src_row * HK, Ti * HK * sizeof(float)},
                {dbt + dst_row * H, beta + src_row * H, (size_t)Ti * H * sizeof(float)}};
            for (const auto &c : cps)
                if ((e = cudaMemcpyAsync(c.dst, c.src, c.bytes, cudaMemcpyHostToDevice, P.h2d)) != cudaSuccess)
                    return cuda_fail(e);
        }
        if ((e = cudaEventRecord(P.in_ready[sl], P.h2d)) != cudaSuccess) return cuda_fail(e);
        // block i on the caller's stream; its output slot was last copied out for block i - 2
        if ((e = cudaStreamWaitEvent(st, P.in_ready[sl], 0)) != cudaSuccess) return cuda_fail(e);
        if (i >= 2 && (e = cudaStreamWaitEvent(st, P.out_done[sl], 0)) != cudaSuccess) return cuda_fail(e);
        const kda_status fs = forward_impl(dq, dk_, dvv, dla, dbt, (i == 0 && !initial_state) ? nullptr : carry,
                                           dout, carry, B, Ti, H, dk, dv, dtype, scale, stream,
                                           kda::KDA_GATE_CHANNEL, L.recs_bytes ? ws + L.recs : nullptr,
                                           L.recs_bytes, 0, T);
        if (fs != KDA_OK) return fs;
        if ((e = cudaEventRecord(P.comp_done[sl], st)) != cudaSuccess) return cuda_fail(e);
        // block i's outputs back to the host
        if ((e = cudaStreamWaitEvent(P.d2h, P.comp_done[sl], 0)) != cudaSuccess) return cuda_fail(e);
        for (int b = 0; b < B; ++b)
            if ((e = cudaMemcpyAsync(out + ((size_t)b * T + t0) * HV, dout + (size_t)b * Ti * HV,
                                     Ti * HV * sizeof(float), cudaMemcpyDeviceToHost, P.d2h)) != cudaSuccess)
                return cuda_fail(e);
        if ((e = cudaEventRecord(P.out_done[sl], P.d2h)) != cudaSuccess) return cuda_fail(e);
    }
    if (final_state &&
        (e = cudaMemcpyAsync(final_state, carry, state_bytes, cudaMemcpyDeviceToHost, P.d2h)) != cudaSuccess)
        return cuda_fail(e);
    // the caller's stream completes after the last copy
    if ((e = cudaEventRecord(P.fin, P.d2h)) != cudaSuccess || (e = cudaStreamWaitEvent(st, P.fin, 0)) != cudaSuccess)
        return cuda_fail(e);
    return KDA_OK;
}

size_t kda_backward_workspace_bytes(int B, int T, int H, int dk, int dv)
{
    if (B <= 0 || H <= 0 || T < 0 || dk != dv || (dk != 64 && dk != 128)) return 0;
    return kda::backward_workspace_bytes(B, T, H, dk);
}

kda_status kda_backward(const void *q, const void *k, const void *v,
                        const float *log_alpha, const float *beta, const float *initial_state,
                        const float *grad_out, const float *grad_final_state,
                        float *grad_q, float *grad_k, float *grad_v, float *grad_log_alpha,
                        float *grad_beta, float *grad_initial_state,
                        int B, int T, int H, int dk, int dv,
                        kda_dtype dtype, float scale, void *workspace, size_t workspace_bytes,
                        void *stream)
{
    g_last_cuda_error[0] = '\0';
    if (B <= 0 || H <= 0 || T < 0 || dk <= 0 || dv <= 0) return KDA_ERR_INVALID_ARG;
    if (dtype != KDA_BF16 && dtype != KDA_F32) return KDA_ERR_INVALID_ARG;
    if (!isfinite(scale)) return KDA_ERR_INVALID_ARG;
    if ((int64_t)B * H * ((int64_t)T + 64) > (int64_t)INT32_MAX) return KDA_ERR_INVALID_ARG;
    if (dk != dv || (dk != 64 && dk != 128)) return KDA_ERR_UNSUPPORTED;
    if (T > 0) {
        if (!q || !k || !v || !log_alpha || !beta || !grad_out || !grad_q || !grad_k || !grad_v ||
            !grad_log_alpha || !grad_beta || !workspace)
            return KDA_ERR_INVALID_ARG;
        if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(log_alpha) || !aligned16(grad_out) ||
            !aligned16(grad_q) || !aligned16(grad_k) || !aligned16(grad_v) || !aligned16(grad_log_alpha) ||
            !aligned4(beta) || !aligned4(grad_beta) || (reinterpret_cast<uintptr_t>(workspace) & 255u))
            return KDA_ERR_MISALIGNED;
        if (workspace_bytes < kda::backward_workspace_bytes(B, T, H, dk)) return KDA_ERR_INVALID_ARG;
    }
    if ((initial_state && !aligned16(initial_state)) || (grad_final_state && !aligned16(grad_final_state)) ||
        (grad_initial_state && !aligned16(grad_initial_state)))
        return KDA_ERR_MISALIGNED;
    if (T == 0 && !grad_initial_state) return KDA_OK;
    kda::BackwardArgs a = {};
    a.q = q; a.k = k; a.v = v; a.log_alpha = log_alpha; a.beta = beta; a.s0 = initial_state;
    a.d_out = grad_out; a.d_final = grad_final_state;
    a.dq = grad_q; a.dk = grad_k; a.dv = grad_v; a.dlog_alpha = grad_log_alpha; a.dbeta = grad_beta;
    a.d_s0 = grad_initial_state;
    a.B = B; a.T = T; a.H = H; a.Dk = dk; a.Dv = dv; a.dtype = dtype;
    a.scale = (scale == 0.0f) ? 1.0f / sqrtf((float)dk) : scale;
    a.workspace = workspace;
    const cudaError_t e = kda::launch_backward(a, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? KDA_OK : cuda_fail(e);
}

kda_status kda_selftest_timeout(unsigned int wait_ms, void *stream)
{
    g_last_cuda_error[0] = '\0';
    if (wait_ms == 0 || wait_ms > 10000) return KDA_ERR_INVALID_ARG;
    cudaError_t e = kda::launch_selftest_timeout(wait_ms, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? KDA_OK : cuda_fail(e);
}

kda_status kda_check_status(void *stream)
{
    g_last_cuda_error[0] = '\0';
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e);
    unsigned int dev_status = 0, gdn_status = 0, split_status = 0;
    e = kda::take_device_status(&dev_status);
    if (e == cudaSuccess) e = kda::take_gdn_device_status(&gdn_status);
    if (e == cudaSuccess) e = kda::take_split_device_status(&split_status);
    if (e != cudaSuccess) return cuda_fail(e);
    return (dev_status | gdn_status | split_status) ? KDA_ERR_TIMEOUT : KDA_OK;
}

}  // extern "C"
