// Chunked KDA prefill on the sm_100a tensor cores (tcgen05 + TMEM), bf16 inputs,
// dk = dv = 128, fp32 state and outputs.
//
// The token step is the one of "Kimi Delta Attention: The Linear Attention
// Behind Kimi K2 and Qwen3", §How Kimi Delta Attention works step by step;
// the sequence is processed chunkwise with the chunk-boundary state as the
// next chunk's initial condition ("KDA Technical Deep Dive", §Systems and
// implementation tradeoffs, Training).  Per (b, h), chunk of c <= 64 tokens,
// entering state S (dk x dv), G_t = in-chunk inclusive sum of log_alpha,
// m = per-channel midpoint of G over the chunk:
//
//   D_AM = [k e^{G-m} ; q e^{G-m}] (k e^{m-G})^T            (128 x 64)
//   A    = Diag(beta) strictly_lower(D_AM[0:64])            A_ij = beta_i k_i.(Gam_i/Gam_j) k_j
//   M    = scale lower(D_AM[64:128])
//   T    = (I + A)^-1  (blocked 16x16 forward substitution, fp32)
//   R    = T Diag(beta),   W = R (k e^G),   Qt = scale q e^G,   Kh = k e^{G_last - G}
//   D1   = [-W ; Qt] S + [R ; M] V          rows 0..63  = Delta = R V - W S
//   D2   = Kh^T Delta,   D1 += [R ; M] (Delta - V)
//                                           rows 64..127 = Qt S + M Delta = O
//   S   <- Diag(e^{G_last}) S + D2
//
// (the M V that the first [R ; M] V product puts into rows 64..127 is cancelled
// by M (Delta - V); both stacked operands stay 128 rows tall, the tcgen05 M).
//
// Precision: the non-input operands need fp32-level accuracy (a single bf16
// rounding of any of them already exceeds a 2e-3 max-abs/rms bar), so every
// fp32 operand X is split X = hi + lo with hi = bf16(X), lo = bf16(X - hi) and
// a product is hi*hi + lo*hi + hi*lo (the lo*lo term is below fp32 rounding);
// V is an exact bf16 input, so its products take two terms.  All MMAs
// accumulate in fp32 in tensor memory.
//
// One CTA (256 threads) owns one (b, h, 32-column value slice): value columns of
// the state evolve independently.  The state slice lives in registers (thread
// (lane dk, half) holds 16 columns of row dk) and is re-split into shared memory
// each chunk as the B operand of the next product.  A chunk whose log-decay
// range is too wide for the split exponentials takes an exact token-by-token
// path on CUDA cores instead.  Every mbarrier wait is bounded; a wait that runs
// out records KDA_ERR_TIMEOUT in a device status word and the CTA exits after
// freeing its tensor memory.
#include "kda_internal.cuh"

namespace kda {

__device__ unsigned int g_kda_device_status;   // bit 0: a bounded wait gave up

namespace {

constexpr int kC = 64, kDK = 128, kDV = 128, kDVS = 32, kNSL = kDV / kDVS, kNT = 256;
constexpr float kGMaxTc = 40.f;
constexpr long long kWaitCycles = 4000000000ll;   // ~2 s at 2 GHz

// ---------------------------------------------------------------- shared memory map
// No-swizzle UMMA tiles: core matrices of 8 rows x 16 bytes.  For a tile indexed
// (outer, inner) the byte offset is core_off(); K-major tiles have outer = M/N,
// inner = K; MN-major tiles have outer = K, inner = M/N.
constexpr uint32_t SM_P = 0;             // [k e^{G-m}; q e^{G-m}] then [-W; Qt]: MN-major 128(K) x 128(M)
constexpr uint32_t SM_P_LO = 32768;
constexpr uint32_t SM_Q = 65536;         // k e^{m-G} (MN-major 128 x 64) then Kh^T (K-major 128 x 64)
constexpr uint32_t SM_Q_LO = SM_Q + 16384;
constexpr uint32_t SM_RM = 98304;        // [R; M] K-major 128(M) x 64(K)
constexpr uint32_t SM_RM_LO = SM_RM + 16384;
constexpr uint32_t SM_W = 131072;        // (k e^G)^T K-major 128 x 64, or fp32 A and T of the solve
constexpr uint32_t SM_W_LO = SM_W + 16384;
constexpr uint32_t SM_AMAT = SM_W;                 // fp32 [64][65]
constexpr uint32_t SM_TMAT = SM_W + 64 * 65 * 4;   // fp32 [64][65]
constexpr uint32_t SM_S = SM_W + 33792;  // state slice, MN-major 128(K) x 32(N)
constexpr uint32_t SM_S_LO = SM_S + 8192;
constexpr uint32_t SM_V = SM_S + 16384;  // value slice, MN-major 64(K) x 32(N), exact bf16
constexpr uint32_t SM_D = SM_V + 4096;   // Delta, MN-major 64 x 32
constexpr uint32_t SM_D_LO = SM_D + 4096;
constexpr uint32_t SM_E = SM_D_LO + 4096;  // Delta - V
constexpr uint32_t SM_E_LO = SM_E + 4096;
constexpr uint32_t SM_BETA = SM_E_LO + 4096;   // fp32 [64]
constexpr uint32_t SM_GAMMA = SM_BETA + 256;    // fp32 [128]
constexpr uint32_t SM_G64 = SM_GAMMA + 512;     // fp64 [2][128]: G_last, midpoint
constexpr uint32_t SM_MBAR = SM_G64 + 2048;     // mbarrier (8 B)
constexpr uint32_t SM_TMEMP = SM_MBAR + 8;      // tensor-memory base address (4 B)
constexpr uint32_t SM_TOTAL = SM_TMEMP + 8;
static_assert(SM_TOTAL <= 227 * 1024, "shared memory");
// token path (wide chunks) reuses [0, SM_W) for fp32 q, k, log_alpha [64][129]
// and the SM_W region for the fp32 state [128][33], v [64][33] and two [8][32] tables.
constexpr int kTP = kDK + 1;

// tile strides (bytes): s_outer, s_inner
constexpr uint32_t P_SO = 2048, P_SI = 128;     // 128 x 128
constexpr uint32_t H_SO = 1024, H_SI = 128;     // 128 x 64  (Q, RM, W tiles)
constexpr uint32_t S_SO = 512, S_SI = 128;      // 128 x 32 / 64 x 32

// tensor-memory columns
constexpr uint32_t TM_AM = 0, TM_W = 64, TM_D1 = 128, TM_D2 = 160, TM_COLS = 256;

__device__ __forceinline__ uint32_t core_off(int outer, int inner, uint32_t so, uint32_t si)
{
    return (uint32_t)(outer >> 3) * so + (uint32_t)(inner >> 3) * si + (uint32_t)(outer & 7) * 16u +
           (uint32_t)(inner & 7) * 2u;
}

// ---------------------------------------------------------------- PTX wrappers
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo)
{
    // no-swizzle shared-memory matrix descriptor (sm_100 format, version 1)
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | ((uint64_t)1 << 46);
}

__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int a_mn, int b_mn)
{
    // D fp32, A bf16, B bf16, dense, no negation
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc)
{
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n"
                 :: "r"(d_tmem), "l"(a), "l"(b), "r"(idesc), "r"(acc) : "memory");
}

__device__ __forceinline__ void umma_commit(uint32_t mbar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 :: "r"(mbar) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void proxy_fence() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16])
{
    uint32_t r[16];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 "
                 "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                   "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
                   "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
                 : "r"(taddr));
    tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32])
{
    float a[16], b[16];
    tmem_ld16(taddr, a);
    tmem_ld16(taddr + 16, b);
#pragma unroll
    for (int i = 0; i < 16; ++i) { v[i] = a[i]; v[16 + i] = b[i]; }
}

__device__ __forceinline__ void mbar_init(uint32_t mbar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(mbar), "r"(count) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Bounded wait for the phase with the given parity; false if it never completed.
__device__ __forceinline__ bool mbar_wait(uint32_t mbar, uint32_t parity)
{
    const long long t0 = clock64();
    for (;;) {
        uint32_t ok;
        asm volatile("{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                     "selp.u32 %0, 1, 0, p;\n\t}\n" : "=r"(ok) : "r"(mbar), "r"(parity) : "memory");
        if (ok) return true;
        if (clock64() - t0 > kWaitCycles) return false;
    }
}

// Split 8 fp32 values into bf16 hi / lo parts packed as two 16-byte vectors.
__device__ __forceinline__ void split8(const float (&x)[8], uint4 &hi, uint4 &lo)
{
    uint32_t h[4], l[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 hv = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
        const float2 hf = __bfloat1622float2(hv);
        const __nv_bfloat162 lv = __floats2bfloat162_rn(x[2 * i] - hf.x, x[2 * i + 1] - hf.y);
        h[i] = *reinterpret_cast<const uint32_t *>(&hv);
        l[i] = *reinterpret_cast<const uint32_t *>(&lv);
    }
    hi = make_uint4(h[0], h[1], h[2], h[3]);
    lo = make_uint4(l[0], l[1], l[2], l[3]);
}

__device__ __forceinline__ void st_split8(uint8_t *smem, uint32_t off_hi, uint32_t off_lo, const float (&x)[8])
{
    uint4 hi, lo;
    split8(x, hi, lo);
    *reinterpret_cast<uint4 *>(smem + off_hi) = hi;
    *reinterpret_cast<uint4 *>(smem + off_lo) = lo;
}

// One product D (+)= A B on split operands.  Terms hi*hi, lo*hi, hi*lo (the last
// only when B has a lo part).  Each term walks K in steps of 16.
__device__ __forceinline__ void mma_split(uint32_t d, uint32_t a_hi, uint32_t a_lo, uint32_t a_lbo,
                                          uint32_t a_sbo, uint32_t b_hi, uint32_t b_lo, uint32_t b_lbo,
                                          uint32_t b_sbo, int ksteps, uint32_t idesc, bool accumulate)
{
    const int nterms = b_lo ? 3 : 2;
    for (int tt = 0; tt < nterms; ++tt) {
        const uint32_t a = (tt == 1) ? a_lo : a_hi;
        const uint32_t b = (tt == 2) ? b_lo : b_hi;
        for (int ks = 0; ks < ksteps; ++ks) {
            const uint64_t ad = smem_desc(a + 2u * a_lbo * ks, a_lbo, a_sbo);
            const uint64_t bd = smem_desc(b + 2u * b_lbo * ks, b_lbo, b_sbo);
            umma_bf16(d, ad, bd, idesc, (accumulate || tt || ks) ? 1u : 0u);
        }
    }
}

// ---------------------------------------------------------------- the kernel
__global__ void __launch_bounds__(kNT, 1)
prefill_tc_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                  const __nv_bfloat16 *__restrict__ v, const float *__restrict__ log_alpha,
                  const float *__restrict__ beta, const float *__restrict__ s0,
                  float *__restrict__ out, float *__restrict__ sT, int T, int H, float scale)
{
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t sbase = (uint32_t)__cvta_generic_to_shared(smem);
    float *sBeta = reinterpret_cast<float *>(smem + SM_BETA);
    float *sGamma = reinterpret_cast<float *>(smem + SM_GAMMA);
    double *sGl = reinterpret_cast<double *>(smem + SM_G64);
    double *sGm = sGl + kDK;
    const uint32_t mbar = sbase + SM_MBAR;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int slice = blockIdx.x % kNSL;
    const int bh = blockIdx.x / kNSL;
    const int b = bh / H, h = bh % H;
    const int col0 = slice * kDVS;
    const int lrow = 32 * (warp & 3) + lane;     // tensor-memory lane this thread reads
    const int half = warp >> 2;                  // which half of the columns it reads

    // ---- tensor memory and the MMA barrier
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     :: "r"(sbase + SM_TMEMP), "r"(TM_COLS) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (tid == 0) mbar_init(mbar, 1);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + SM_TMEMP);
    const uint32_t tlane = (uint32_t)(32 * (warp & 3)) << 16;
    uint32_t phase = 0;
    bool failed = false;

    // ---- state slice: thread holds row lrow, columns 16*half .. +15
    float S[16];
    {
        const int n0 = 16 * half;
#pragma unroll
        for (int j = 0; j < 16; ++j)
            S[j] = s0 ? s0[((size_t)bh * kDK + lrow) * kDV + col0 + n0 + j] : 0.f;
    }
    auto write_state_tile = [&]() {
#pragma unroll
        for (int g = 0; g < 2; ++g) {
            float x[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) x[e] = S[8 * g + e];
            const uint32_t off = core_off(lrow, 16 * half + 8 * g, S_SO, S_SI);
            st_split8(smem, SM_S + off, SM_S_LO + off, x);
        }
    };
    write_state_tile();

    const int nchunks = (T + kC - 1) / kC;
    for (int n = 0; n < nchunks && !failed; ++n) {
        const int t0 = n * kC;
        const int c = min(kC, T - t0);
        auto gk = [&](int t, int ch) { return (((size_t)b * T + t0 + t) * H + h) * kDK + ch; };
        auto gv = [&](int t) { return (((size_t)b * T + t0 + t) * H + h) * kDV + col0; };

        // ---- stage beta and the value slice (exact bf16, MN-major 64 x 32)
        if (tid < kC) sBeta[tid] = (tid < c) ? beta[((size_t)b * T + t0 + tid) * H + h] : 0.f;
        {
            const int t = tid >> 2, g = tid & 3;
            uint4 val = make_uint4(0u, 0u, 0u, 0u);
            if (t < c) val = *reinterpret_cast<const uint4 *>(v + gv(t) + 8 * g);
            *reinterpret_cast<uint4 *>(smem + SM_V + core_off(t, 8 * g, S_SO, S_SI)) = val;
        }

        // ---- pass 1 (thread per key channel): fp64 log-decay sums, range, path choice
        bool wide = false;
        if (tid < kDK) {
            double run = 0.0, lo = 0.0, hi = 0.0;
            for (int t = 0; t < c; ++t) {
                run += (double)log_alpha[gk(t, tid)];
                lo = (t == 0) ? run : fmin(lo, run);
                hi = (t == 0) ? run : fmax(hi, run);
            }
            sGl[tid] = run;
            sGm[tid] = 0.5 * (hi + lo);
            wide = !(0.5 * (hi - lo) <= (double)kGMaxTc && fabs(hi) <= 2.0 * kGMaxTc &&
                     fabs(lo) <= 2.0 * kGMaxTc);
        }
        const bool token_path = __syncthreads_or(wide) != 0;

        if (!token_path) {
            // ---- pass 2: [k e^{G-m}; q e^{G-m}] (SM_P) and k e^{m-G} (SM_Q), hi/lo
            if (tid < kDK) {
                const int ch = tid;
                const double m = sGm[ch];
                double run = 0.0;
                for (int g = 0; g < 8; ++g) {
                    float kr[8], qr[8], kb[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int t = 8 * g + e;
                        float kk = 0.f, qq = 0.f;
                        if (t < c) {
                            run += (double)log_alpha[gk(t, ch)];
                            kk = __bfloat162float(k[gk(t, ch)]);
                            qq = __bfloat162float(q[gk(t, ch)]);
                        }
                        const float x = (float)(run - m);
                        const float up = __expf(x), dn = __expf(-x);
                        kr[e] = kk * up; qr[e] = qq * up; kb[e] = kk * dn;
                    }
                    const uint32_t o1 = core_off(ch, 8 * g, P_SO, P_SI);
                    const uint32_t o2 = core_off(ch, 64 + 8 * g, P_SO, P_SI);
                    const uint32_t o3 = core_off(ch, 8 * g, H_SO, H_SI);
                    st_split8(smem, SM_P + o1, SM_P_LO + o1, kr);
                    st_split8(smem, SM_P + o2, SM_P_LO + o2, qr);
                    st_split8(smem, SM_Q + o3, SM_Q_LO + o3, kb);
                }
            }
            proxy_fence();
            __syncthreads();
            if (tid == 0) {
                tc_fence_after();
                mma_split(tmem + TM_AM, sbase + SM_P, sbase + SM_P_LO, P_SO, P_SI,
                          sbase + SM_Q, sbase + SM_Q_LO, H_SO, H_SI, kDK / 16,
                          idesc_bf16(128, 64, 1, 1), false);
                umma_commit(mbar);
            }
            failed = __syncthreads_or(!mbar_wait(mbar, phase)) != 0;
            phase ^= 1;
            if (failed) break;
            tc_fence_after();

            // ---- A (fp32, rows 0..63) to the solve; M (rows 64..127) into [R; M]
            {
                float x[32];
                tmem_ld32(tmem + tlane + TM_AM + 32 * half, x);
                if (lrow < 64) {
                    const int i = lrow;
                    float *Am = reinterpret_cast<float *>(smem + SM_AMAT) + i * 65;
                    const float bi = sBeta[i];
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const int j = 32 * half + e;
                        Am[j] = (j < i) ? bi * x[e] : 0.f;
                    }
                } else {
                    const int i = lrow - 64;
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        float y[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int j = 32 * half + 8 * g + e;
                            y[e] = (j <= i) ? scale * x[8 * g + e] : 0.f;
                        }
                        const uint32_t o = core_off(lrow, 32 * half + 8 * g, H_SO, H_SI);
                        st_split8(smem, SM_RM + o, SM_RM_LO + o, y);
                    }
                }
            }
            __syncthreads();

            // ---- T = (I + A)^-1, blocked 16 x 16, fp32
            {
                const float *Am = reinterpret_cast<const float *>(smem + SM_AMAT);
                float *Tm = reinterpret_cast<float *>(smem + SM_TMAT);
                if (tid < 64) {
                    // diagonal blocks by forward substitution, one column per thread
                    const int blk = tid >> 4, j = tid & 15, o = 16 * blk;
                    float x[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        float s = (i == j) ? 1.f : 0.f;
                        if (i > j) {
#pragma unroll
                            for (int l = 0; l < i; ++l)
                                if (l >= j) s -= Am[(o + i) * 65 + o + l] * x[l];
                        }
                        x[i] = s;
                    }
#pragma unroll
                    for (int i = 0; i < 16; ++i) Tm[(o + i) * 65 + o + j] = x[i];
                }
                __syncthreads();
                for (int dd = 1; dd < 4; ++dd) {
                    // Y_ab = sum_{c=b}^{a-1} A_ac T_cb, kept in the unused upper block (b, a)
                    for (int e = tid; e < (4 - dd) * 256; e += kNT) {
                        const int a = dd + e / 256, bb = a - dd;
                        const int i = (e & 255) >> 4, j = e & 15;
                        float s = 0.f;
                        for (int cb = bb; cb < a; ++cb)
#pragma unroll
                            for (int l = 0; l < 16; ++l)
                                s += Am[(16 * a + i) * 65 + 16 * cb + l] * Tm[(16 * cb + l) * 65 + 16 * bb + j];
                        Tm[(16 * bb + i) * 65 + 16 * a + j] = s;
                    }
                    __syncthreads();
                    // T_ab = -T_aa Y_ab
                    for (int e = tid; e < (4 - dd) * 256; e += kNT) {
                        const int a = dd + e / 256, bb = a - dd;
                        const int i = (e & 255) >> 4, j = e & 15;
                        float s = 0.f;
#pragma unroll
                        for (int l = 0; l < 16; ++l)
                            if (l <= i) s += Tm[(16 * a + i) * 65 + 16 * a + l] * Tm[(16 * bb + l) * 65 + 16 * a + j];
                        Tm[(16 * a + i) * 65 + 16 * bb + j] = -s;
                    }
                    __syncthreads();
                }
                // R = T Diag(beta) into rows 0..63 of [R; M]
                for (int id = tid; id < 512; id += kNT) {
                    const int i = id >> 3, jg = id & 7;
                    float y[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int j = 8 * jg + e;
                        y[e] = (j <= i) ? Tm[i * 65 + j] * sBeta[j] : 0.f;
                    }
                    const uint32_t o = core_off(i, 8 * jg, H_SO, H_SI);
                    st_split8(smem, SM_RM + o, SM_RM_LO + o, y);
                }
            }
            __syncthreads();

            // ---- pass 3: (k e^G)^T (SM_W), scale q e^G (SM_P rows 64..), Kh^T (SM_Q), Gamma
            if (tid < kDK) {
                const int ch = tid;
                const double gl = sGl[ch];
                double run = 0.0;
                for (int g = 0; g < 8; ++g) {
                    float kt[8], qt[8], kh[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int t = 8 * g + e;
                        float kk = 0.f, qq = 0.f;
                        if (t < c) {
                            run += (double)log_alpha[gk(t, ch)];
                            kk = __bfloat162float(k[gk(t, ch)]);
                            qq = __bfloat162float(q[gk(t, ch)]);
                        }
                        const float eg = __expf((float)run), el = __expf((float)(gl - run));
                        kt[e] = kk * eg; qt[e] = scale * qq * eg; kh[e] = kk * el;
                    }
                    const uint32_t ow = core_off(ch, 8 * g, H_SO, H_SI);
                    const uint32_t oq = core_off(ch, 64 + 8 * g, P_SO, P_SI);
                    st_split8(smem, SM_W + ow, SM_W_LO + ow, kt);
                    st_split8(smem, SM_P + oq, SM_P_LO + oq, qt);
                    st_split8(smem, SM_Q + ow, SM_Q_LO + ow, kh);
                }
                sGamma[ch] = (float)exp(gl);
            }
            proxy_fence();
            __syncthreads();
            if (tid == 0) {
                tc_fence_after();
                // W^T = (k e^G)^T R^T  -> TM_W (rows dk, columns token)
                mma_split(tmem + TM_W, sbase + SM_W, sbase + SM_W_LO, H_SI, H_SO,
                          sbase + SM_RM, sbase + SM_RM_LO, H_SI, H_SO, kC / 16,
                          idesc_bf16(128, 64, 0, 0), false);
                umma_commit(mbar);
            }
            failed = __syncthreads_or(!mbar_wait(mbar, phase)) != 0;
            phase ^= 1;
            if (failed) break;
            tc_fence_after();

            // ---- -W into rows 0..63 of SM_P (MN-major: outer dk, inner token)
            {
                float x[32];
                tmem_ld32(tmem + tlane + TM_W + 32 * half, x);
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    float y[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) y[e] = -x[8 * g + e];
                    const uint32_t o = core_off(lrow, 32 * half + 8 * g, P_SO, P_SI);
                    st_split8(smem, SM_P + o, SM_P_LO + o, y);
                }
            }
            proxy_fence();
            tc_fence_before();
            __syncthreads();
            if (tid == 0) {
                tc_fence_after();
                // D1 = [-W; Qt] S + [R; M] V
                mma_split(tmem + TM_D1, sbase + SM_P, sbase + SM_P_LO, P_SO, P_SI,
                          sbase + SM_S, sbase + SM_S_LO, S_SO, S_SI, kDK / 16,
                          idesc_bf16(128, kDVS, 1, 1), false);
                mma_split(tmem + TM_D1, sbase + SM_RM, sbase + SM_RM_LO, H_SI, H_SO,
                          sbase + SM_V, 0u, S_SO, S_SI, kC / 16,
                          idesc_bf16(128, kDVS, 0, 1), true);
                umma_commit(mbar);
            }
            failed = __syncthreads_or(!mbar_wait(mbar, phase)) != 0;
            phase ^= 1;
            if (failed) break;
            tc_fence_after();

            // ---- Delta (rows 0..63 of D1) and Delta - V as split B operands
            if (lrow < 64) {
                float x[16];
                tmem_ld16(tmem + tlane + TM_D1 + 16 * half, x);
                const int t = lrow;
#pragma unroll
                for (int g = 0; g < 2; ++g) {
                    const uint32_t o = core_off(t, 16 * half + 8 * g, S_SO, S_SI);
                    const uint4 vv = *reinterpret_cast<const uint4 *>(smem + SM_V + o);
                    const __nv_bfloat16 *vb = reinterpret_cast<const __nv_bfloat16 *>(&vv);
                    float d[8], ev[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        d[e] = x[8 * g + e];
                        ev[e] = d[e] - __bfloat162float(vb[e]);
                    }
                    st_split8(smem, SM_D + o, SM_D_LO + o, d);
                    st_split8(smem, SM_E + o, SM_E_LO + o, ev);
                }
            }
            proxy_fence();
            tc_fence_before();
            __syncthreads();
            if (tid == 0) {
                tc_fence_after();
                // D2 = Kh^T Delta;  D1 += [R; M] (Delta - V)
                mma_split(tmem + TM_D2, sbase + SM_Q, sbase + SM_Q_LO, H_SI, H_SO,
                          sbase + SM_D, sbase + SM_D_LO, S_SO, S_SI, kC / 16,
                          idesc_bf16(128, kDVS, 0, 1), false);
                mma_split(tmem + TM_D1, sbase + SM_RM, sbase + SM_RM_LO, H_SI, H_SO,
                          sbase + SM_E, sbase + SM_E_LO, S_SO, S_SI, kC / 16,
                          idesc_bf16(128, kDVS, 0, 1), true);
                umma_commit(mbar);
            }
            failed = __syncthreads_or(!mbar_wait(mbar, phase)) != 0;
            phase ^= 1;
            if (failed) break;
            tc_fence_after();

            // ---- state update and outputs
            {
                float x[16];
                tmem_ld16(tmem + tlane + TM_D2 + 16 * half, x);
                const float gm = sGamma[lrow];
#pragma unroll
                for (int j = 0; j < 16; ++j) S[j] = gm * S[j] + x[j];
                write_state_tile();
                if (lrow >= 64) {
                    const int t = lrow - 64;
                    float o[16];
                    tmem_ld16(tmem + tlane + TM_D1 + 16 * half, o);
                    if (t < c) {
                        float4 *dst = reinterpret_cast<float4 *>(out + gv(t) + 16 * half);
#pragma unroll
                        for (int g = 0; g < 4; ++g)
                            dst[g] = make_float4(o[4 * g], o[4 * g + 1], o[4 * g + 2], o[4 * g + 3]);
                    }
                }
            }
            proxy_fence();
            tc_fence_before();
            __syncthreads();
        } else {
            // ---- exact token-by-token path for a chunk with a very wide decay range
            float *fq = reinterpret_cast<float *>(smem);
            float *fk = fq + kC * kTP;
            float *fa = fk + kC * kTP;
            float *fS = reinterpret_cast<float *>(smem + SM_W);     // [128][33]
            float *fv = fS + kDK * 33;                                // [64][33]
            float *red = fv + kC * 33;                                // [2][8][32]
            for (int idx = tid; idx < kC * kDK; idx += kNT) {
                const int t = idx / kDK, ch = idx % kDK;
                float qq = 0.f, kk = 0.f, la = 0.f;
                if (t < c) {
                    qq = __bfloat162float(q[gk(t, ch)]);
                    kk = __bfloat162float(k[gk(t, ch)]);
                    la = log_alpha[gk(t, ch)];
                }
                fq[t * kTP + ch] = qq; fk[t * kTP + ch] = kk; fa[t * kTP + ch] = la;
            }
            for (int idx = tid; idx < kC * kDVS; idx += kNT) {
                const int t = idx / kDVS, x = idx % kDVS;
                fv[t * 33 + x] = (t < c) ? __bfloat162float(v[gv(t) + x]) : 0.f;
            }
#pragma unroll
            for (int j = 0; j < 16; ++j) fS[lrow * 33 + 16 * half + j] = S[j];
            __syncthreads();
            constexpr int RG = kNT / kDVS, RPT = kDK / RG;
            const int x = tid % kDVS, rg = tid / kDVS;
            float sreg[RPT];
#pragma unroll
            for (int r = 0; r < RPT; ++r) sreg[r] = fS[(rg * RPT + r) * 33 + x];
            for (int t = 0; t < c; ++t) {
                float pk = 0.f;
#pragma unroll
                for (int r = 0; r < RPT; ++r) {
                    const int ch = rg * RPT + r;
                    sreg[r] *= expf(fa[t * kTP + ch]);
                    pk += sreg[r] * fk[t * kTP + ch];
                }
                red[rg * kDVS + x] = pk;
                __syncthreads();
                float p = 0.f;
#pragma unroll
                for (int j = 0; j < RG; ++j) p += red[j * kDVS + x];
                const float d = sBeta[t] * (fv[t * 33 + x] - p);
                float pq = 0.f;
#pragma unroll
                for (int r = 0; r < RPT; ++r) {
                    const int ch = rg * RPT + r;
                    sreg[r] += fk[t * kTP + ch] * d;
                    pq += sreg[r] * fq[t * kTP + ch];
                }
                red[RG * kDVS + rg * kDVS + x] = pq;
                __syncthreads();
                if (rg == 0) {
                    float o = 0.f;
#pragma unroll
                    for (int j = 0; j < RG; ++j) o += red[RG * kDVS + j * kDVS + x];
                    out[gv(t) + x] = scale * o;
                }
                __syncthreads();
            }
#pragma unroll
            for (int r = 0; r < RPT; ++r) fS[(rg * RPT + r) * 33 + x] = sreg[r];
            __syncthreads();
#pragma unroll
            for (int j = 0; j < 16; ++j) S[j] = fS[lrow * 33 + 16 * half + j];
            write_state_tile();
            proxy_fence();
            __syncthreads();
        }
    }

    if (failed) {
        if (tid == 0) atomicOr(&g_kda_device_status, 1u);
    } else if (sT) {
        float4 *dst = reinterpret_cast<float4 *>(sT + ((size_t)bh * kDK + lrow) * kDV + col0 + 16 * half);
#pragma unroll
        for (int g = 0; g < 4; ++g) dst[g] = make_float4(S[4 * g], S[4 * g + 1], S[4 * g + 2], S[4 * g + 3]);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem), "r"(TM_COLS) : "memory");
    }
}

}  // namespace

bool prefill_tc_supported(const ForwardArgs &a)
{
    return a.dtype == KDA_BF16 && a.dk == kDK && a.dv == kDV;
}

cudaError_t launch_prefill_tc(const ForwardArgs &a, cudaStream_t stream)
{
    cudaError_t e = cudaFuncSetAttribute(prefill_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SM_TOTAL);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)((size_t)a.B * a.H * kNSL);
    prefill_tc_kernel<<<grid, kNT, SM_TOTAL, stream>>>(
        static_cast<const __nv_bfloat16 *>(a.q), static_cast<const __nv_bfloat16 *>(a.k),
        static_cast<const __nv_bfloat16 *>(a.v), a.log_alpha, a.beta, a.s0, a.out, a.sT, a.T, a.H,
        a.scale);
    e = cudaGetLastError();
    if (e == cudaSuccess) note_launch();
    return e;
}

cudaError_t take_device_status(unsigned int *status)
{
    unsigned int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbol(status, g_kda_device_status, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    if (*status) e = cudaMemcpyToSymbol(g_kda_device_status, &zero, sizeof(unsigned int));
    return e;
}

}  // namespace kda
