// Chunked KDA prefill on CUDA cores, fp32 arithmetic throughout.
//
// The pages give the token step ("Kimi Delta Attention: The Linear Attention
// Behind Kimi K2 and Qwen3", §How Kimi Delta Attention works step by step) and
// say production kernels process the sequence chunkwise, the state at a chunk
// boundary being the initial condition of the next chunk ("KDA Technical Deep
// Dive", §Systems and implementation tradeoffs, Training).  This kernel is the
// re-association of the token step over a chunk of C = 64 tokens (the WY / UT
// form).  Per (b, h), chunk of c <= 64 tokens, entering state S (dk x dv):
//
//   G_t  = sum_{s<=t} log_alpha_s (per key channel, reset every chunk)
//   m    = per-channel midpoint of G over the chunk (a reference point that
//          keeps every exponential below exp(range/2))
//   A_ij = beta_i sum_c k_ic k_jc exp(G_ic - G_jc)      j <  i
//   M_ij = scale  sum_c q_ic k_jc exp(G_ic - G_jc)      j <= i
//          (each exp split as exp(G_i - m) * exp(m - G_j))
//   [W | U] = (I + A)^-1 Diag(beta) [k*exp(G) | V]      (forward substitution)
//   D    = U - W S                    (row t = the error e_t of the token step)
//   O    = (scale q*exp(G)) S + M D
//   S   <- Diag(exp(G_last)) S + (k*exp(G_last - G))^T D
//
// A chunk whose log-decay range in some channel is too wide for the split
// exponentials to stay finite (range > 2 * kGMax) is processed token by token
// with the plain step instead; nothing is clamped.
//
// One CTA owns one (b, h, value slice of kDVS columns) and walks the chunks in
// order with its state slice resident in shared memory.  Value columns of the
// state evolve independently, so slices need no communication; the
// chunk-local products A, M, W are recomputed per slice.
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kC = kChunk;
constexpr int kThreads = 256;
constexpr int kDVS = 32;             // value columns per CTA
constexpr float kGMax = 40.f;        // largest |exponent| allowed in a split factor

template <int DK>
struct SimtSmem {
    static constexpr int P = DK + 1;     // padded pitch of [C][DK] tiles
    static constexpr int PV = kDVS + 1;  // padded pitch of [*][DVS] tiles
    static constexpr int PC = kC + 1;    // padded pitch of [C][C] tiles
    static constexpr int off_q = 0;
    static constexpr int off_k = off_q + kC * P;
    static constexpr int off_x = off_k + kC * P;
    static constexpr int off_y = off_x + kC * P;
    static constexpr int off_v = off_y + kC * P;
    static constexpr int off_a = off_v + kC * PV;
    static constexpr int off_m = off_a + kC * PC;
    static constexpr int off_s = off_m + kC * PC;
    static constexpr int off_d = off_s + DK * PV;
    static constexpr int off_o = off_d + kC * PV;
    static constexpr int off_b = off_o + kC * PV;
    static constexpr int off_gl = off_b + kC;
    static constexpr int off_red = off_gl + DK;           // [2][8][DVS] reduction tables
    static constexpr int off_g64 = (off_red + 2 * 8 * kDVS + 1) & ~1;   // [2][DK] doubles
    static constexpr int total = off_g64 + 4 * DK;
    static constexpr size_t bytes = sizeof(float) * (size_t)total;
};

template <int DK, int DV, typename InT>
__global__ void __launch_bounds__(kThreads, 1)
prefill_simt_kernel(const InT *__restrict__ q, const InT *__restrict__ k,
                    const InT *__restrict__ v, const float *__restrict__ log_alpha,
                    const float *__restrict__ beta, const float *__restrict__ s0,
                    float *__restrict__ out, float *__restrict__ sT,
                    int T, int H, float scale, int gate)
{
    using L = SimtSmem<DK>;
    constexpr int P = L::P, PV = L::PV, PC = L::PC;
    constexpr int NS = DV / kDVS;
    extern __shared__ float sm[];
    float *sQ = sm + L::off_q, *sK = sm + L::off_k, *sX = sm + L::off_x, *sY = sm + L::off_y;
    float *sV = sm + L::off_v, *sA = sm + L::off_a, *sM = sm + L::off_m, *sS = sm + L::off_s;
    float *sD = sm + L::off_d, *sO = sm + L::off_o, *sB = sm + L::off_b;
    float *sGl = sm + L::off_gl, *sRed = sm + L::off_red;
    double *sGl64 = reinterpret_cast<double *>(sm + L::off_g64), *sGm64 = sGl64 + DK;

    const int tid = threadIdx.x;
    const int slice = blockIdx.x % NS;
    const int bh = blockIdx.x / NS;
    const int b = bh / H, h = bh % H;
    const int col0 = slice * kDVS;

    // ---- initial state slice
    for (int idx = tid; idx < DK * kDVS; idx += kThreads) {
        const int r = idx / kDVS, x = idx % kDVS;
        sS[r * PV + x] = s0 ? s0[((size_t)bh * DK + r) * DV + col0 + x] : 0.f;
    }

    const int nchunks = (T + kC - 1) / kC;
    for (int n = 0; n < nchunks; ++n) {
        const int t0 = n * kC;
        const int c = min(kC, T - t0);
        __syncthreads();   // previous chunk fully consumed

        // ---- stage v and beta (rows past c are zero: they change nothing)
        for (int idx = tid; idx < kC * kDVS; idx += kThreads) {
            const int t = idx / kDVS, x = idx % kDVS;
            sV[t * PV + x] = (t < c) ? to_f32(v[(((size_t)b * T + t0 + t) * H + h) * DV + col0 + x]) : 0.f;
        }
        if (tid < kC) sB[tid] = (tid < c) ? beta[((size_t)b * T + t0 + tid) * H + h] : 0.f;
        // global index of (token t of this chunk, key channel ch)
        auto gk = [&](int t, int ch) { return (((size_t)b * T + t0 + t) * H + h) * DK + ch; };
        // log_alpha of (token t, key channel ch): per channel, one per token and head, or none
        auto la_at = [&](int t, int ch) -> float {
            if (gate == KDA_GATE_CHANNEL) return log_alpha[gk(t, ch)];
            if (gate == KDA_GATE_SCALAR) return log_alpha[((size_t)b * T + t0 + t) * H + h];
            return 0.f;
        };

        // ---- pass 1, one thread per key channel: the in-chunk log-decay sums in
        // fp64 (so each exponent argument below carries a single rounding) and
        // their range, which decides between the factored and the token path
        bool wide = false;
        if (tid < DK) {
            double run = 0.0, lo = 0.0, hi = 0.0;
            for (int t = 0; t < c; ++t) {
                run += (double)la_at(t, tid);
                lo = (t == 0) ? run : fmin(lo, run);
                hi = (t == 0) ? run : fmax(hi, run);
            }
            sGl64[tid] = run;
            sGm64[tid] = 0.5 * (hi + lo);
            wide = !(0.5 * (hi - lo) <= (double)kGMax && fabs(hi) <= 2.0 * kGMax && fabs(lo) <= 2.0 * kGMax);
        }
        const bool token_path = __syncthreads_or(wide) != 0;

        if (!token_path) {
            // ---- pass 2: split exponentials around the per-channel midpoint m
            if (tid < DK) {
                const double m = sGm64[tid];
                double run = 0.0;
                for (int t = 0; t < kC; ++t) {
                    float kk = 0.f, qq = 0.f;
                    if (t < c) {
                        run += (double)la_at(t, tid);
                        kk = to_f32(k[gk(t, tid)]);
                        qq = to_f32(q[gk(t, tid)]);
                    }
                    const float up = expf((float)(run - m)), dn = expf((float)(m - run));
                    sX[t * P + tid] = kk * up;            // k exp(G - m)
                    sY[t * P + tid] = kk * dn;            // k exp(m - G)
                    sQ[t * P + tid] = qq * up;            // q exp(G - m)
                }
            }
            __syncthreads();

            // ---- A (strictly lower, times beta_i) and M (lower, times scale): 4x4 per thread
            {
                const int ib = tid / 16, jb = tid % 16;
                const int i0 = ib * 4, j0 = jb * 4;
                float acc_a[4][4] = {}, acc_m[4][4] = {};
                if (jb <= ib) {
                    for (int ch = 0; ch < DK; ++ch) {
                        float xa[4], xq[4], yb[4];
#pragma unroll
                        for (int r = 0; r < 4; ++r) {
                            xa[r] = sX[(i0 + r) * P + ch];
                            xq[r] = sQ[(i0 + r) * P + ch];
                            yb[r] = sY[(j0 + r) * P + ch];
                        }
#pragma unroll
                        for (int r = 0; r < 4; ++r)
#pragma unroll
                            for (int s = 0; s < 4; ++s) {
                                acc_a[r][s] += xa[r] * yb[s];
                                acc_m[r][s] += xq[r] * yb[s];
                            }
                    }
                }
#pragma unroll
                for (int r = 0; r < 4; ++r)
#pragma unroll
                    for (int s = 0; s < 4; ++s) {
                        const int i = i0 + r, j = j0 + s;
                        sA[i * PC + j] = (j < i) ? sB[i] * acc_a[r][s] : 0.f;
                        sM[i * PC + j] = (j <= i) ? scale * acc_m[r][s] : 0.f;
                    }
            }
            __syncthreads();

            // ---- pass 3: right-hand sides beta*k*exp(G) (into sK), scale*q*exp(G)
            //      (sQ), k*exp(G_last - G) (sY), beta*v (sV); Gamma = exp(G_last)
            if (tid < DK) {
                const double gl = sGl64[tid];
                double run = 0.0;
                for (int t = 0; t < kC; ++t) {
                    float kk = 0.f, qq = 0.f;
                    if (t < c) {
                        run += (double)la_at(t, tid);
                        kk = to_f32(k[gk(t, tid)]);
                        qq = to_f32(q[gk(t, tid)]);
                    }
                    const float eg = expf((float)run), el = expf((float)(gl - run));
                    sK[t * P + tid] = sB[t] * kk * eg;
                    sQ[t * P + tid] = scale * qq * eg;
                    sY[t * P + tid] = kk * el;
                }
                sGl[tid] = (float)exp(gl);
            }
            for (int idx = tid; idx < kC * kDVS; idx += kThreads) {
                const int t = idx / kDVS, x = idx % kDVS;
                sV[t * PV + x] *= sB[t];
            }
            __syncthreads();

            // ---- [W | U] = (I + A)^-1 [beta k exp(G) | beta V], one column per thread
            if (tid < DK + kDVS) {
                float *colp = (tid < DK) ? (sK + tid) : (sV + (tid - DK));
                const int pitch = (tid < DK) ? P : PV;
                for (int i = 1; i < kC; ++i) {
                    float x = colp[i * pitch];
                    const float *arow = sA + i * PC;
                    for (int j = 0; j < i; ++j) x -= arow[j] * colp[j * pitch];
                    colp[i * pitch] = x;
                }
            }
            __syncthreads();

            // ---- D = U - W S and Pq = (scale q exp(G)) S: rows ti*8..+7, column x
            {
                const int x = tid % kDVS, ti = tid / kDVS;
                float dacc[8], pacc[8];
#pragma unroll
                for (int r = 0; r < 8; ++r) { dacc[r] = 0.f; pacc[r] = 0.f; }
                for (int ch = 0; ch < DK; ++ch) {
                    const float sv = sS[ch * PV + x];
#pragma unroll
                    for (int r = 0; r < 8; ++r) {
                        dacc[r] += sK[(ti * 8 + r) * P + ch] * sv;
                        pacc[r] += sQ[(ti * 8 + r) * P + ch] * sv;
                    }
                }
#pragma unroll
                for (int r = 0; r < 8; ++r) {
                    const int i = ti * 8 + r;
                    sD[i * PV + x] = sV[i * PV + x] - dacc[r];
                    sO[i * PV + x] = pacc[r];
                }
            }
            __syncthreads();

            // ---- O += M D (causal), S <- exp(G_last) S + Kh^T D
            {
                const int x = tid % kDVS, ti = tid / kDVS;
                float oacc[8];
#pragma unroll
                for (int r = 0; r < 8; ++r) oacc[r] = sO[(ti * 8 + r) * PV + x];
                for (int j = 0; j < ti * 8 + 8; ++j) {
                    const float dj = sD[j * PV + x];
#pragma unroll
                    for (int r = 0; r < 8; ++r) oacc[r] += sM[(ti * 8 + r) * PC + j] * dj;
                }
#pragma unroll
                for (int r = 0; r < 8; ++r) sO[(ti * 8 + r) * PV + x] = oacc[r];

                constexpr int RPT = DK / (kThreads / kDVS);      // state rows per thread
                float sacc[RPT];
#pragma unroll
                for (int r = 0; r < RPT; ++r) {
                    const int ch = ti * RPT + r;
                    sacc[r] = sGl[ch] * sS[ch * PV + x];
                }
                for (int j = 0; j < kC; ++j) {
                    const float dj = sD[j * PV + x];
#pragma unroll
                    for (int r = 0; r < RPT; ++r) sacc[r] += sY[j * P + ti * RPT + r] * dj;
                }
                __syncthreads();   // every read of the old state is done
#pragma unroll
                for (int r = 0; r < RPT; ++r) sS[(ti * RPT + r) * PV + x] = sacc[r];
            }
            __syncthreads();
        } else {
            // ---- token-by-token path for a chunk with a very wide decay range.
            // Stage raw q, k, log_alpha; thread (rg, x) owns rows rg*RPT..+RPT-1, column x.
            for (int idx = tid; idx < kC * DK; idx += kThreads) {
                const int t = idx / DK, ch = idx % DK;
                float qq = 0.f, kk = 0.f, la = 0.f;
                if (t < c) { qq = to_f32(q[gk(t, ch)]); kk = to_f32(k[gk(t, ch)]); la = la_at(t, ch); }
                sQ[t * P + ch] = qq; sK[t * P + ch] = kk; sX[t * P + ch] = la;
            }
            __syncthreads();
            constexpr int RG = kThreads / kDVS;                  // row groups (8)
            constexpr int RPT = DK / RG;
            const int x = tid % kDVS, rg = tid / kDVS;
            float sreg[RPT];
#pragma unroll
            for (int r = 0; r < RPT; ++r) sreg[r] = sS[(rg * RPT + r) * PV + x];
            for (int t = 0; t < c; ++t) {
                float pk = 0.f;
#pragma unroll
                for (int r = 0; r < RPT; ++r) {
                    const int ch = rg * RPT + r;
                    sreg[r] *= expf(sX[t * P + ch]);
                    pk += sreg[r] * sK[t * P + ch];
                }
                sRed[rg * kDVS + x] = pk;
                __syncthreads();
                float p = 0.f;
#pragma unroll
                for (int j = 0; j < RG; ++j) p += sRed[j * kDVS + x];
                const float d = sB[t] * (sV[t * PV + x] - p);
                float pq = 0.f;
#pragma unroll
                for (int r = 0; r < RPT; ++r) {
                    const int ch = rg * RPT + r;
                    sreg[r] += sK[t * P + ch] * d;
                    pq += sreg[r] * sQ[t * P + ch];
                }
                sRed[RG * kDVS + rg * kDVS + x] = pq;
                __syncthreads();
                if (rg == 0) {
                    float o = 0.f;
#pragma unroll
                    for (int j = 0; j < RG; ++j) o += sRed[RG * kDVS + j * kDVS + x];
                    sO[t * PV + x] = scale * o;
                }
                __syncthreads();   // the reduction table is reused by the next token
            }
#pragma unroll
            for (int r = 0; r < RPT; ++r) sS[(rg * RPT + r) * PV + x] = sreg[r];
            __syncthreads();
        }

        // ---- write the chunk's outputs
        for (int idx = tid; idx < c * kDVS; idx += kThreads) {
            const int t = idx / kDVS, x = idx % kDVS;
            out[(((size_t)b * T + t0 + t) * H + h) * DV + col0 + x] = sO[t * PV + x];
        }
    }

    if (sT) {
        __syncthreads();
        for (int idx = tid; idx < DK * kDVS; idx += kThreads) {
            const int r = idx / kDVS, x = idx % kDVS;
            sT[((size_t)bh * DK + r) * DV + col0 + x] = sS[r * PV + x];
        }
    }
}

template <int DK, int DV, typename InT>
cudaError_t launch_typed(const ForwardArgs &a, cudaStream_t stream)
{
    auto kern = prefill_simt_kernel<DK, DV, InT>;
    const size_t smem = SimtSmem<DK>::bytes;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)((size_t)a.B * a.H * (DV / kDVS));
    kern<<<grid, kThreads, smem, stream>>>(
        static_cast<const InT *>(a.q), static_cast<const InT *>(a.k),
        static_cast<const InT *>(a.v), a.log_alpha, a.beta, a.s0, a.out, a.sT,
        a.T, a.H, a.scale, a.gate);
    cudaError_t e2 = cudaGetLastError();
    if (e2 == cudaSuccess) note_launch();
    return e2;
}

template <typename InT>
cudaError_t launch_dims(const ForwardArgs &a, cudaStream_t stream)
{
    if (a.dk == 128 && a.dv == 128) return launch_typed<128, 128, InT>(a, stream);
    if (a.dk == 64 && a.dv == 64) return launch_typed<64, 64, InT>(a, stream);
    if (a.dk == 128 && a.dv == 64) return launch_typed<128, 64, InT>(a, stream);
    if (a.dk == 64 && a.dv == 128) return launch_typed<64, 128, InT>(a, stream);
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_prefill_simt(const ForwardArgs &a, cudaStream_t stream)
{
    if (a.dtype == KDA_BF16) return launch_dims<__nv_bfloat16>(a, stream);
    return launch_dims<float>(a, stream);
}

}  // namespace kda
