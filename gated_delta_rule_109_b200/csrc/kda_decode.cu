// Single-token KDA decode step (one token per sequence, state updated in place).
//
// "KDA Technical Deep Dive", §Systems and implementation tradeoffs, Decoding:
// each new token costs one state update plus one query-state product,
// independent of the context length; the state is updated in place
// (§How the Kimi gate changes memory).  Step order as in "Kimi Delta
// Attention: The Linear Attention Behind Kimi K2 and Qwen3", §How Kimi Delta
// Attention works step by step: decay per key channel, predict, error, write,
// read after the write.
//
// Per head the whole update is one pass over the fp32 state held in
// registers:
//     S~ = Diag(alpha) S
//     p  = S~^T k,  r = S~^T q          (both reductions over key channels)
//     d  = beta (v - p)
//     S  = S~ + k d^T                   (written back in place)
//     o  = scale (r + (k.q) d)          (= scale S^T q after the write)
// The state (dk*dv*4 bytes read and written per head) is all the traffic that
// matters, so the kernel is shaped for HBM: 16-byte coalesced loads issued
// up front, every state element touched once, reductions through shuffles
// and a small shared-memory table.
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kDecodeThreads = 256;

// PER_CHANNEL: log_alpha is [B, H, dk] (KDA); otherwise [B, H] or null (one
// decay for all channels, or none).  NS CTAs share a head, each with DV / NS of its
// value columns (columns of the state never mix, so they need no communication).
template <int DK, int DV, typename InT, bool PER_CHANNEL, int NS>
__global__ void __launch_bounds__(kDecodeThreads, NS == 1 ? 2 : 3)
decode_step_kernel(const InT *__restrict__ q, const InT *__restrict__ k,
                   const InT *__restrict__ v, const float *__restrict__ log_alpha,
                   const float *__restrict__ beta, float *__restrict__ state,
                   float *__restrict__ out, float scale)
{
    constexpr int CGH = DV / 4;                // float4 column groups per state row
    constexpr int CG = CGH / NS;               // ... handled by this CTA
    constexpr int RS = kDecodeThreads / CG;    // row stride between a thread's rows
    constexpr int RPT = DK / RS;               // state rows held per thread
    static_assert(RPT * RS == DK && CG * RS == kDecodeThreads, "shape");

    __shared__ float4 red_p[RS][CG];
    __shared__ float4 red_r[RS][CG];
    __shared__ float s_kq;

    // Programmatic dependent launch: once every CTA of this step has started, the next
    // step may be launched, so that its CTAs take the SM slots this step's last wave
    // frees instead of waiting for the launch after it completes.  Nothing is read
    // before the kernel ahead on the stream (the previous step, or whatever produced
    // this step's inputs) has completed and its writes are visible.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");

    const int bh = blockIdx.x / NS;            // b * H + h
    const int tid = threadIdx.x;
    const int cg = (blockIdx.x % NS) * CG + tid % CG;   // column group within the head
    const int r0 = tid / CG;

    float4 *S = reinterpret_cast<float4 *>(state) + (size_t)bh * DK * CGH;
    float4 s[RPT];
#pragma unroll
    for (int i = 0; i < RPT; ++i) s[i] = __ldcs(&S[(r0 + i * RS) * CGH + cg]);

    const InT *qh = q + (size_t)bh * DK;
    const InT *kh = k + (size_t)bh * DK;
    // decay of this head: per key channel (lah), or one value for all channels
    const float *lah = log_alpha + (size_t)bh * DK;
    const float a_all = (!PER_CHANNEL && log_alpha) ? expf(log_alpha[bh]) : 1.f;

    // k.q for the read after the write (warp 0)
    if (tid < 32) {
        float acc = 0.f;
        for (int c = tid; c < DK; c += 32) acc += to_f32(kh[c]) * to_f32(qh[c]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (tid == 0) s_kq = acc;
    }

    float kr[RPT];
    float4 pp = make_float4(0.f, 0.f, 0.f, 0.f), rr = pp;
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const int r = r0 + i * RS;
        const float a = PER_CHANNEL ? expf(lah[r]) : a_all;
        const float kc = to_f32(kh[r]);
        const float qc = to_f32(qh[r]);
        kr[i] = kc;
        s[i].x *= a; s[i].y *= a; s[i].z *= a; s[i].w *= a;
        pp.x += kc * s[i].x; pp.y += kc * s[i].y; pp.z += kc * s[i].z; pp.w += kc * s[i].w;
        rr.x += qc * s[i].x; rr.y += qc * s[i].y; rr.z += qc * s[i].z; rr.w += qc * s[i].w;
    }
    red_p[r0][tid % CG] = pp;
    red_r[r0][tid % CG] = rr;
    __syncthreads();

    float4 p = make_float4(0.f, 0.f, 0.f, 0.f), r = p;
#pragma unroll
    for (int j = 0; j < RS; ++j) {
        const float4 a = red_p[j][tid % CG], b = red_r[j][tid % CG];
        p.x += a.x; p.y += a.y; p.z += a.z; p.w += a.w;
        r.x += b.x; r.y += b.y; r.z += b.z; r.w += b.w;
    }
    const InT *vh = v + (size_t)bh * DV + 4 * cg;
    const float bt = beta[bh];
    float4 d;
    d.x = bt * (to_f32(vh[0]) - p.x);
    d.y = bt * (to_f32(vh[1]) - p.y);
    d.z = bt * (to_f32(vh[2]) - p.z);
    d.w = bt * (to_f32(vh[3]) - p.w);

#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const float kc = kr[i];
        s[i].x += kc * d.x; s[i].y += kc * d.y; s[i].z += kc * d.z; s[i].w += kc * d.w;
        __stcs(&S[(r0 + i * RS) * CGH + cg], s[i]);
    }
    if (r0 == 0) {
        const float kq = s_kq;
        float4 o;
        o.x = scale * (r.x + kq * d.x);
        o.y = scale * (r.y + kq * d.y);
        o.z = scale * (r.z + kq * d.z);
        o.w = scale * (r.w + kq * d.w);
        reinterpret_cast<float4 *>(out)[(size_t)bh * CGH + cg] = o;
    }
}

#ifndef KDA_DECODE_SPLIT
#define KDA_DECODE_SPLIT 2
#endif

template <int DK, int DV, typename InT>
cudaError_t launch_typed(const DecodeArgs &a, cudaStream_t stream)
{
    // two CTAs per head when a head has 128 value columns (half the registers per
    // thread, four CTAs per SM), else one
    constexpr int NS = (DV == 128) ? KDA_DECODE_SPLIT : 1;
    const unsigned grid = (unsigned)((size_t)a.B * a.H * NS);
    auto kernel = (a.gate == KDA_GATE_CHANNEL) ? decode_step_kernel<DK, DV, InT, true, NS>
                                               : decode_step_kernel<DK, DV, InT, false, NS>;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kDecodeThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e2 = cudaLaunchKernelEx(&cfg, kernel, static_cast<const InT *>(a.q), static_cast<const InT *>(a.k),
                                        static_cast<const InT *>(a.v), a.log_alpha, a.beta, a.state, a.out,
                                        a.scale);
    if (e2 == cudaSuccess) e2 = cudaGetLastError();
    if (e2 == cudaSuccess) note_launch();
    return e2;
}

template <typename InT>
cudaError_t launch_dims(const DecodeArgs &a, cudaStream_t stream)
{
    if (a.dk == 128 && a.dv == 128) return launch_typed<128, 128, InT>(a, stream);
    if (a.dk == 64 && a.dv == 64) return launch_typed<64, 64, InT>(a, stream);
    if (a.dk == 128 && a.dv == 64) return launch_typed<128, 64, InT>(a, stream);
    if (a.dk == 64 && a.dv == 128) return launch_typed<64, 128, InT>(a, stream);
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t stream)
{
    if (a.dtype == KDA_BF16) return launch_dims<__nv_bfloat16>(a, stream);
    return launch_dims<float>(a, stream);
}

}  // namespace kda
