// The KDA backward pass: gradients of the forward with respect to q, k, v,
// log_alpha, beta and the initial state, given the cotangents of the outputs
// and of the final state.
//
// The pages define the forward by its token step ("Kimi Delta Attention: The
// Linear Attention Behind Kimi K2 and Qwen3", §How Kimi Delta Attention works
// step by step) and name chunkwise training without giving a gradient ("KDA
// Technical Deep Dive", §Systems and implementation tradeoffs, Training).  The
// backward here is the reverse-mode derivative of that step.  Per token, with
// a = exp(log_alpha_t):
//
//   forward   S~ = Diag(a) S,  p = S~^T k,  e = beta (v - p),  S' = S~ + k e^T,  o = scale S'^T q
//   backward  (dS = dL/dS', swept from the last token to the first)
//             dS += scale q dO^T;          dq = scale S' dO
//             de = dS^T k;  dv = beta de;  dbeta = de . (v - p);  dp = -beta de
//             dk = dS e + S~ dp;           dS~ = dS + k dp^T
//             dlog_alpha = rowsum(dS~ * S~);  dS <- Diag(a) dS~
//
// Value columns of S never mix, so every pass is parallel over columns: warp w of
// a CTA owns one column, lane l owns the key rows l, l + 32, ...  Sums over rows
// (p and dS^T k, which feed the recurrence) are warp sums; sums over columns (dq,
// dk, dlog_alpha) are outputs only and are reduced across warps in shared memory.
//
// Three kernels, all fp32 on CUDA cores:
//   bwd_state_kernel     the forward state before every 8th token (checkpoints)
//   bwd_adjoint_kernel   dS at the end of every chunk of 64 tokens (and dL/dS_0),
//                        swept backwards
//   bwd_chunk_grad_kernel  one CTA per (b, h, chunk): per group of 8 tokens, the
//                        states recomputed from the group's checkpoint and the
//                        backward swept from the chunk's end adjoint, one
//                        value-column block after another; the chunk's rows of dq,
//                        dk, dlog_alpha and dbeta belong to this CTA alone, so the
//                        blocks accumulate into them without atomics.
// Saved states and adjoints are column-major per (b, h): [slot][b, h][column][row],
// so a warp (one column, rows across lanes) reads and writes 128-byte rows.
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kBC = 64;              // tokens per chunk
constexpr int kBW = 16;              // warps per CTA = value columns per block
constexpr int kBThreads = kBW * 32;
constexpr int kSub = 8;              // tokens between recomputation checkpoints

__device__ __forceinline__ float warp_sum(float x)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// L2 prefetch of a global range (16-byte aligned, a multiple of 16 bytes); a hint
// that nothing waits for
__device__ __forceinline__ void l2_prefetch(const void *src, uint32_t bytes)
{
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" :: "l"(src), "r"(bytes) : "memory");
}

__device__ __forceinline__ void cp_async(void *dst, const void *src, int bytes, bool valid)
{
    const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst);
    if (bytes == 16)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" :: "r"(d), "l"(src), "r"(valid ? 16 : 0)
                     : "memory");
    else
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" :: "r"(d), "l"(src), "r"(valid ? 4 : 0)
                     : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;" :: "n"(N) : "memory"); }

// R consecutive row values of one token as fp32 (one 8- or 16-byte shared load)
template <int R>
__device__ __forceinline__ void ld_rows(const float *p, float (&o)[R])
{
    if constexpr (R == 4) {
        const float4 x = *reinterpret_cast<const float4 *>(p);
        o[0] = x.x; o[1] = x.y; o[2] = x.z; o[3] = x.w;
    } else {
        const float2 x = *reinterpret_cast<const float2 *>(p);
        o[0] = x.x; o[1] = x.y;
    }
}
template <int R>
__device__ __forceinline__ void ld_rows(const __nv_bfloat16 *p, float (&o)[R])
{
    if constexpr (R == 4) {
        const uint2 x = *reinterpret_cast<const uint2 *>(p);
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&x.x));
        const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&x.y));
        o[0] = a.x; o[1] = a.y; o[2] = b.x; o[3] = b.y;
    } else {
        const uint32_t x = *reinterpret_cast<const uint32_t *>(p);
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&x));
        o[0] = a.x; o[1] = a.y;
    }
}
template <int R>
__device__ __forceinline__ void st_rows(float *p, const float (&x)[R])
{
    if constexpr (R == 4)
        *reinterpret_cast<float4 *>(p) = make_float4(x[0], x[1], x[2], x[3]);
    else
        *reinterpret_cast<float2 *>(p) = make_float2(x[0], x[1]);
}

// One chunk's per-token inputs in shared memory (rows past the sequence end are
// zero-filled): key rows (and query rows) in the input dtype, log_alpha rows,
// beta, and the block's 8 value (and output-cotangent) columns.
template <typename Tin, int D, bool WITH_Q = true>
struct Stage {
    Tin k[kBC][D];
    Tin q[WITH_Q ? kBC : 1][D];
    float la[kBC][D];                      // log_alpha as staged, then alpha = exp(log_alpha)
    Tin v[kBC][kBW];
    float dout[WITH_Q ? kBC : 1][kBW];
    float beta[kBC];
};

struct Dims {
    int T, H, nc;
    float scale;
};

__device__ __forceinline__ size_t tok_row(int b, int t, int h, const Dims &d)
{
    return ((size_t)b * d.T + t) * d.H + h;
}

// Copies the chunk's key rows (and query rows), log_alpha rows and beta into a
// stage (cp.async; rows past the sequence end zero-filled, their source clamped to
// a valid row).
template <typename Tin, int D, bool WITH_Q>
__device__ void stage_rows(Stage<Tin, D, WITH_Q> &s, const Tin *k, const Tin *q, const float *la,
                           const float *beta, int b, int h, int c, const Dims &d)
{
    const int tid = threadIdx.x, t0 = c * kBC;
    constexpr int kPerRowK = D * (int)sizeof(Tin) / 16, kPerRowA = D * 4 / 16;
    for (int i = tid; i < kBC * kPerRowK; i += kBThreads) {
        const int t = i / kPerRowK, j = i % kPerRowK;
        const bool ok = t0 + t < d.T;
        const size_t row = tok_row(b, ok ? t0 + t : 0, h, d);
        cp_async(reinterpret_cast<uint8_t *>(&s.k[t][0]) + 16 * j,
                 reinterpret_cast<const uint8_t *>(k + row * D) + 16 * j, 16, ok);
        if (WITH_Q)
            cp_async(reinterpret_cast<uint8_t *>(&s.q[t][0]) + 16 * j,
                     reinterpret_cast<const uint8_t *>(q + row * D) + 16 * j, 16, ok);
    }
    for (int i = tid; i < kBC * kPerRowA; i += kBThreads) {
        const int t = i / kPerRowA, j = i % kPerRowA;
        const bool ok = t0 + t < d.T;
        cp_async(&s.la[t][4 * j], la + tok_row(b, ok ? t0 + t : 0, h, d) * D + 4 * j, 16, ok);
    }
    if (tid < kBC) {
        const bool ok = t0 + tid < d.T;
        cp_async(&s.beta[tid], beta + tok_row(b, ok ? t0 + tid : 0, h, d), 4, ok);
    }
}

// Copies the chunk's value columns col0 .. col0 + kBW - 1 (and output-cotangent columns).
template <typename Tin, int D, bool WITH_Q>
__device__ void stage_cols(Stage<Tin, D, WITH_Q> &s, const Tin *v, const float *dout, int b, int h, int c,
                           int col0, const Dims &d)
{
    const int tid = threadIdx.x, t0 = c * kBC;
    constexpr int kPerRowV = kBW * (int)sizeof(Tin) / 16;    // 1 (bf16) or 2 (fp32)
    for (int i = tid; i < kBC * kPerRowV; i += kBThreads) {
        const int t = i / kPerRowV, j = i % kPerRowV;
        const bool ok = t0 + t < d.T;
        cp_async(reinterpret_cast<uint8_t *>(&s.v[t][0]) + 16 * j,
                 reinterpret_cast<const uint8_t *>(v + tok_row(b, ok ? t0 + t : 0, h, d) * D + col0) + 16 * j, 16, ok);
    }
    if (WITH_Q) {
        constexpr int kPerRowO = kBW * 4 / 16;
        for (int i = tid; i < kBC * kPerRowO; i += kBThreads) {
            const int t = i / kPerRowO, j = i % kPerRowO;
            const bool ok = t0 + t < d.T;
            cp_async(&s.dout[t][4 * j], dout + tok_row(b, ok ? t0 + t : 0, h, d) * D + col0 + 4 * j, 16, ok);
        }
    }
}

// log_alpha rows of a landed stage -> alpha = exp(log_alpha), once per chunk
// (every warp of the CTA reads the same rows).
template <typename Tin, int D, bool WITH_Q>
__device__ __forceinline__ void stage_exp(Stage<Tin, D, WITH_Q> &s)
{
    float *x = &s.la[0][0];
    for (int i = threadIdx.x; i < kBC * D; i += kBThreads) x[i] = expf(x[i]);
}

// ---------------------------------------------------------------- forward states
// CTA (b, h, block of value columns); writes S before every 8th token:
// states[t / 8][b, h][col][row].
template <typename Tin, int D>
__global__ void __launch_bounds__(kBThreads)
bwd_state_kernel(const Tin *__restrict__ k, const Tin *__restrict__ v, const float *__restrict__ la,
                 const float *__restrict__ beta, const float *__restrict__ s0, float *__restrict__ states, Dims d)
{
    constexpr int R = D / 32;
    extern __shared__ __align__(16) uint8_t smem[];
    using St = Stage<Tin, D, false>;
    St *st = reinterpret_cast<St *>(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rb = R * lane;                   // this lane's rows: rb .. rb + R - 1
    const int nblk = D / kBW;
    const int blk = blockIdx.x % nblk, bh = blockIdx.x / nblk;
    const int b = bh / d.H, h = bh % d.H;
    const int col = blk * kBW + warp;
    float S[R];
#pragma unroll
    for (int i = 0; i < R; ++i) S[i] = s0 ? s0[((size_t)bh * D + rb + i) * D + col] : 0.f;
    auto stage = [&](int c) {
        stage_rows<Tin, D, false>(st[c & 1], k, nullptr, la, beta, b, h, c, d);
        stage_cols<Tin, D, false>(st[c & 1], v, nullptr, b, h, c, blk * kBW, d);
        cp_commit();
    };
    if (d.nc > 0) stage(0);
    for (int c = 0; c < d.nc; ++c) {
        St &s = st[c & 1];
        if (c + 1 < d.nc) {
            stage(c + 1);
            cp_wait<1>();
        } else {
            cp_wait<0>();
        }
        __syncthreads();
        stage_exp(s);
        __syncthreads();
        const int len = min(kBC, d.T - c * kBC);
        for (int t = 0; t < len; ++t) {
            if (t % kSub == 0)
                st_rows<R>(states + (((size_t)(c * kBC + t) / kSub * (gridDim.x / nblk) + bh) * D + col) * D + rb, S);
            float part = 0.f, kk[R], aa[R];
            ld_rows<R>(&s.k[t][rb], kk);
            ld_rows<R>(&s.la[t][rb], aa);
#pragma unroll
            for (int i = 0; i < R; ++i) {
                S[i] *= aa[i];
                part += S[i] * kk[i];
            }
            const float p = warp_sum(part);
            const float e = s.beta[t] * (to_f32(s.v[t][warp]) - p);
#pragma unroll
            for (int i = 0; i < R; ++i) S[i] += kk[i] * e;
        }
        __syncthreads();      // the stage is refilled two chunks later
    }
}

// ---------------------------------------------------------------- adjoint states
// CTA (b, h, block of 8 value columns); sweeps the tokens backwards from dS =
// d_final (or 0) and writes dS at the end of every chunk: dstates[c][b, h][col][row];
// at the start of the sequence, dL/dS_0 into d_s0 (if given).
template <typename Tin, int D>
__global__ void __launch_bounds__(kBThreads)
bwd_adjoint_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
                   const float *__restrict__ la, const float *__restrict__ beta, const float *__restrict__ dout,
                   const float *__restrict__ d_final, float *__restrict__ dstates, float *__restrict__ d_s0, Dims d)
{
    constexpr int R = D / 32;
    extern __shared__ __align__(16) uint8_t smem[];
    using St = Stage<Tin, D, true>;
    St *st = reinterpret_cast<St *>(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rb = R * lane;                   // this lane's rows: rb .. rb + R - 1
    const int nblk = D / kBW;
    const int blk = blockIdx.x % nblk, bh = blockIdx.x / nblk;
    const int b = bh / d.H, h = bh % d.H;
    const int col = blk * kBW + warp;
    float dS[R];
#pragma unroll
    for (int i = 0; i < R; ++i) dS[i] = d_final ? d_final[((size_t)bh * D + rb + i) * D + col] : 0.f;
    auto stage = [&](int c) {
        stage_rows<Tin, D, true>(st[c & 1], k, q, la, beta, b, h, c, d);
        stage_cols<Tin, D, true>(st[c & 1], v, dout, b, h, c, blk * kBW, d);
        cp_commit();
    };
    if (d.nc > 0) stage(d.nc - 1);
    for (int c = d.nc - 1; c >= 0; --c) {
        St &s = st[c & 1];
        if (c > 0) {
            stage(c - 1);
            cp_wait<1>();
        } else {
            cp_wait<0>();
        }
        __syncthreads();
        stage_exp(s);
        __syncthreads();
        st_rows<R>(dstates + (((size_t)c * (gridDim.x / nblk) + bh) * D + col) * D + rb, dS);
        const int len = min(kBC, d.T - c * kBC);
        for (int t = len - 1; t >= 0; --t) {
            const float go = d.scale * s.dout[t][warp];
            float part = 0.f, kk[R], qq[R], aa[R];
            ld_rows<R>(&s.k[t][rb], kk);
            ld_rows<R>(&s.q[t][rb], qq);
            ld_rows<R>(&s.la[t][rb], aa);
#pragma unroll
            for (int i = 0; i < R; ++i) {
                dS[i] += qq[i] * go;
                part += dS[i] * kk[i];
            }
            const float dp = -s.beta[t] * warp_sum(part);
#pragma unroll
            for (int i = 0; i < R; ++i) dS[i] = aa[i] * (dS[i] + kk[i] * dp);
        }
        __syncthreads();
    }
    if (d_s0) {
#pragma unroll
        for (int i = 0; i < R; ++i) d_s0[((size_t)bh * D + rb + i) * D + col] = dS[i];
    }
}

// ---------------------------------------------------------------- per-chunk gradients
template <typename Tin, int D>
struct GradSmem {
    Stage<Tin, D, true> s;                 // k, q, log_alpha, beta of the chunk; v, dO of the block
    float red[2][kBW][3][D];               // per-warp partials of dq, dk, dlog_alpha (two tokens in turn)
    float redb[2][kBW];                    // ... and of dbeta
};

template <typename Tin, int D>
__global__ void __launch_bounds__(kBThreads, 1)
bwd_chunk_grad_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
                      const float *__restrict__ la, const float *__restrict__ beta, const float *__restrict__ dout,
                      const float *__restrict__ states, const float *__restrict__ dstates,
                      float *__restrict__ dq, float *__restrict__ dk, float *__restrict__ dv,
                      float *__restrict__ dla, float *__restrict__ dbeta, Dims d)
{
    constexpr int R = D / 32;
    extern __shared__ __align__(16) uint8_t smem[];
    GradSmem<Tin, D> &g = *reinterpret_cast<GradSmem<Tin, D> *>(smem);
    Stage<Tin, D, true> &s = g.s;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int rb = R * lane;                   // this lane's rows: rb .. rb + R - 1
    const int c = blockIdx.x % d.nc, bh = blockIdx.x / d.nc;
    const int b = bh / d.H, h = bh % d.H;
    const int t0 = c * kBC, len = min(kBC, d.T - t0);
    const size_t BH = (size_t)gridDim.x / d.nc;
    const float *dSe = dstates + ((size_t)c * BH + bh) * D * D;

    for (int blk = 0; blk < D / kBW; ++blk) {
        const int col = blk * kBW + warp;
        // warm L2 with the next column block's end adjoint and group checkpoints (the
        // first block also with its own, while the chunk is staged): they come from
        // DRAM, and this CTA is alone on its SM, so nothing else hides their latency
        if (warp == 0) {
            const int ng = (len - 1) / kSub + 1;
            for (int pbk = (blk == 0 ? 0 : blk + 1); pbk <= blk + 1 && pbk < D / kBW; ++pbk) {
                const size_t c0 = (size_t)pbk * kBW * D;
                if (lane < ng)
                    l2_prefetch(states + ((size_t)(t0 / kSub + lane) * BH + bh) * D * D + c0, kBW * D * 4);
                else if (lane == 31)
                    l2_prefetch(dSe + c0, kBW * D * 4);
            }
        }
        // the chunk's rows are staged once, the block's value and cotangent columns every block
        if (blk == 0) stage_rows<Tin, D, true>(s, k, q, la, beta, b, h, c, d);
        stage_cols<Tin, D, true>(s, v, dout, b, h, c, blk * kBW, d);
        cp_commit();
        cp_wait<0>();
        __syncthreads();
        if (blk == 0) {
            stage_exp(s);
            __syncthreads();
        }

        // ---- backward sweep, one group of 8 tokens at a time (states recomputed from its checkpoint)
        float dS[R];
#pragma unroll
        for (int i = 0; i < R; ++i) dS[i] = dSe[(size_t)col * D + rb + i];   // column-major: contiguous
        for (int j = (len - 1) / kSub; j >= 0; --j) {
            float Sb[kSub][R], pb[kSub], eb[kSub];
            float X[R];
            ld_rows<R>(states + (((size_t)(t0 / kSub + j) * BH + bh) * D + col) * D + rb, X);
#pragma unroll
            for (int u = 0; u < kSub; ++u) {
                const int t = j * kSub + u;
#pragma unroll
                for (int i = 0; i < R; ++i) Sb[u][i] = X[i];
                pb[u] = eb[u] = 0.f;
                if (t < len) {
                    float part = 0.f, kk[R], aa[R];
                    ld_rows<R>(&s.k[t][rb], kk);
                    ld_rows<R>(&s.la[t][rb], aa);
#pragma unroll
                    for (int i = 0; i < R; ++i) {
                        X[i] *= aa[i];
                        part += X[i] * kk[i];
                    }
                    pb[u] = warp_sum(part);
                    eb[u] = s.beta[t] * (to_f32(s.v[t][warp]) - pb[u]);
#pragma unroll
                    for (int i = 0; i < R; ++i) X[i] += kk[i] * eb[u];
                }
            }
#pragma unroll
            for (int u = kSub - 1; u >= 0; --u) {
                const int t = j * kSub + u;
                if (t >= len) continue;
                const int buf = t & 1;                      // partials buffer of this token
                const size_t row = ((size_t)b * d.T + t0 + t) * d.H + h;
                // the accumulated sums of the previous column blocks, fetched early
                float prev[(3 * D + 1 + kBThreads - 1) / kBThreads];
#pragma unroll
                for (int m = 0; m < (3 * D + 1 + kBThreads - 1) / kBThreads; ++m) {
                    const int idx = tid + m * kBThreads;
                    prev[m] = 0.f;
                    if (blk > 0 && idx < 3 * D + 1)
                        prev[m] = idx < 3 * D ? (idx < D ? dq : idx < 2 * D ? dk : dla)[row * D + idx % D]
                                              : dbeta[row];
                }
                const float bt = s.beta[t], go = d.scale * s.dout[t][warp];
                float a[R], kk[R], qq[R], St[R], w0[R], w1[R], w2[R], part = 0.f;
                ld_rows<R>(&s.la[t][rb], a);
                ld_rows<R>(&s.k[t][rb], kk);
                ld_rows<R>(&s.q[t][rb], qq);
#pragma unroll
                for (int i = 0; i < R; ++i) {
                    St[i] = a[i] * Sb[u][i];                       // S~
                    w0[i] = (St[i] + kk[i] * eb[u]) * go;          // dq share: S' (after the write) dO
                    dS[i] += qq[i] * go;
                    part += dS[i] * kk[i];
                }
                st_rows<R>(&g.red[buf][warp][0][rb], w0);
                const float de = warp_sum(part);
                const float dp = -bt * de;
#pragma unroll
                for (int i = 0; i < R; ++i) {
                    w1[i] = dS[i] * eb[u] + St[i] * dp;            // dk share
                    const float dSt = dS[i] + kk[i] * dp;          // dS~
                    w2[i] = dSt * St[i];                           // dlog_alpha share
                    dS[i] = a[i] * dSt;
                }
                st_rows<R>(&g.red[buf][warp][1][rb], w1);
                st_rows<R>(&g.red[buf][warp][2][rb], w2);
                if (lane == 0) {
                    g.redb[buf][warp] = de * (to_f32(s.v[t][warp]) - pb[u]);
                    dv[row * D + col] = bt * de;
                }
                // one barrier per token: buffer buf is written again two tokens later,
                // after the next token's barrier, by which time every thread has read it
                __syncthreads();
#pragma unroll
                for (int m = 0; m < (3 * D + 1 + kBThreads - 1) / kBThreads; ++m) {
                    const int idx = tid + m * kBThreads;
                    if (idx < 3 * D) {
                        const int qn = idx / D, r = idx % D;
                        float sum = prev[m];
#pragma unroll
                        for (int w = 0; w < kBW; ++w) sum += g.red[buf][w][qn][r];
                        (qn == 0 ? dq : qn == 1 ? dk : dla)[row * D + r] = sum;
                    } else if (idx == 3 * D) {
                        float sum = prev[m];
#pragma unroll
                        for (int w = 0; w < kBW; ++w) sum += g.redb[buf][w];
                        dbeta[row] = sum;
                    }
                }
            }
        }
        __syncthreads();      // the next block re-stages v and dO
    }
}

template <typename Tin, int D>
cudaError_t launch_backward_t(const BackwardArgs &a, cudaStream_t stream)
{
    const Tin *q = static_cast<const Tin *>(a.q), *k = static_cast<const Tin *>(a.k),
              *v = static_cast<const Tin *>(a.v);
    Dims d;
    d.T = a.T;
    d.H = a.H;
    d.nc = (a.T + kBC - 1) / kBC;
    d.scale = a.scale;
    const size_t BH = (size_t)a.B * a.H;
    float *states = reinterpret_cast<float *>(a.workspace);
    float *dstates = states + (size_t)((a.T + kSub - 1) / kSub) * BH * D * D;
    const unsigned col_ctas = (unsigned)(BH * (D / kBW));
    const size_t stage_s = 2 * sizeof(Stage<Tin, D, false>), stage2 = 2 * sizeof(Stage<Tin, D, true>);
    cudaError_t e = cudaSuccess;
    if (d.nc > 0) {
        e = cudaFuncSetAttribute(bwd_state_kernel<Tin, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)stage_s);
        if (e != cudaSuccess) return e;
        bwd_state_kernel<Tin, D><<<col_ctas, kBThreads, stage_s, stream>>>(k, v, a.log_alpha, a.beta, a.s0, states, d);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        note_launch();
    }
    e = cudaFuncSetAttribute(bwd_adjoint_kernel<Tin, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)stage2);
    if (e != cudaSuccess) return e;
    bwd_adjoint_kernel<Tin, D><<<col_ctas, kBThreads, stage2, stream>>>(q, k, v, a.log_alpha, a.beta, a.d_out,
                                                                          a.d_final, dstates, a.d_s0, d);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    note_launch();
    if (d.nc > 0) {
        const size_t sm = sizeof(GradSmem<Tin, D>);
        e = cudaFuncSetAttribute(bwd_chunk_grad_kernel<Tin, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        if (e != cudaSuccess) return e;
        bwd_chunk_grad_kernel<Tin, D><<<(unsigned)(BH * d.nc), kBThreads, sm, stream>>>(
            q, k, v, a.log_alpha, a.beta, a.d_out, states, dstates, a.dq, a.dk, a.dv, a.dlog_alpha, a.dbeta, d);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        note_launch();
    }
    return cudaSuccess;
}

}  // namespace

size_t backward_workspace_bytes(int B, int T, int H, int D)
{
    const size_t nc = ((size_t)T + kBC - 1) / kBC, ns = ((size_t)T + kSub - 1) / kSub;
    return (ns + nc) * (size_t)B * H * D * D * sizeof(float);
}

cudaError_t launch_backward(const BackwardArgs &a, cudaStream_t stream)
{
    if (a.dtype == KDA_BF16)
        return a.Dk == 128 ? launch_backward_t<__nv_bfloat16, 128>(a, stream)
                           : launch_backward_t<__nv_bfloat16, 64>(a, stream);
    return a.Dk == 128 ? launch_backward_t<float, 128>(a, stream) : launch_backward_t<float, 64>(a, stream);
}

}  // namespace kda
