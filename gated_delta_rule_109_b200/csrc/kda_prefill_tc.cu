// Chunked KDA prefill on the sm_100a tensor cores (tcgen05 + TMEM), bf16 inputs,
// dk = dv = 128, fp32 state and outputs.
//
// The token step is the one of "Kimi Delta Attention: The Linear Attention
// Behind Kimi K2 and Qwen3", §How Kimi Delta Attention works step by step;
// the sequence is processed chunkwise with the chunk-boundary state as the
// next chunk's initial condition ("KDA Technical Deep Dive", §Systems and
// implementation tradeoffs, Training).  Per (b, h), chunk of c <= 64 tokens,
// entering state S (dk x dv), G_t = in-chunk inclusive sum of log_alpha and
// m = per-channel midpoint of G over the chunk:
//
//   Kr = k e^{G-m},  Qr = scale q e^{G-m},  Kb = k e^{m-G},  S' = Diag(e^m) S
//   D    = [Kr ; Qr] [Kb | S']                                     (128 x 96, one product)
//          columns 0..63:  A = Diag(beta) strictly_lower(D[0:64]),  M = lower(D[64:128])
//          columns 64..95: rows 0..63 = k e^G S (= K~ S),  rows 64..127 = scale q e^G S (= Q~ S)
//   T    = (I + A)^-1  (blocked forward substitution, fp32),  R = T Diag(beta)
//   E    = V - K~ S,   Delta = R E       (row t of Delta is the delta-rule error e_t)
//   O    = Q~ S + M Delta,   with M Delta = M E + M (Delta - E)
//   S   <- Diag(e^{G_last}) S + Diag(e^{G_last - m}) Kb^T Delta
//
// A_ij = beta_i k_i.(Gamma_i/Gamma_j) k_j and (I + A)^-1 are the WY/UT
// quantities of the chunkwise delta rule.  Three tensor-core round trips per
// chunk: D; [R; M] E; and (Kb^T Delta, [R; M] (Delta - E)).  The stacked [R; M]
// keeps every product 128 rows tall (the tcgen05 M); its M E half is cancelled
// by the M (Delta - E) of the last round trip.
//
// Precision: the non-input operands need fp32-level accuracy (a single bf16
// rounding of any of them already exceeds a 2e-3 max-abs/rms bar), so every
// fp32 operand X is split X = hi + lo with hi = bf16(X), lo = bf16(X - hi) and
// a product is hi*hi + lo*hi + hi*lo (lo*lo is below fp32 rounding).
// Accumulation is fp32 in tensor memory.
//
// One CTA (256 threads) owns one (b, h, 32-column value slice): value columns
// of the state evolve independently.  The state slice stays in registers
// (thread (lane dk, half) holds 16 columns of row dk).  Each chunk's q, k and
// log_alpha rows are staged in shared memory by cp.async.bulk copies issued
// one chunk ahead.  A chunk whose log-decay range is too wide for the split
// exponentials takes an exact token-by-token path on CUDA cores.  Every
// mbarrier wait is bounded; a wait that runs out records KDA_ERR_TIMEOUT in a
// device status word and the CTA exits after freeing its tensor memory.
#include "kda_tc_ptx.cuh"

namespace kda {

__device__ unsigned int g_kda_device_status;   // bit 0: a bounded wait gave up

namespace {

using namespace tcx;

constexpr int kC = 64, kDK = 128, kDV = 128, kDVS = 32, kNSL = kDV / kDVS, kNT = 256;
constexpr int kNB = 64 + kDVS;                     // N of the first product
constexpr float kGMaxTc = 40.f;

// ---------------------------------------------------------------- shared memory map
// No-swizzle UMMA tiles: core matrices of 8 rows x 16 bytes.  For a tile indexed
// (outer, inner) the byte offset is core_off(); K-major tiles have outer = M/N,
// inner = K; MN-major tiles have outer = K, inner = M/N.
constexpr uint32_t SM_P = 0;             // [Kr; Qr]: outer dk, inner row 0..127
constexpr uint32_t SM_P_LO = 32768;
constexpr uint32_t SM_B = 65536;         // [Kb | S']: outer dk, inner 0..63 token, 64..95 state column
constexpr uint32_t SM_B_LO = SM_B + 24576;
constexpr uint32_t SM_RM = SM_B_LO + 24576;   // [R; M]: outer row 0..127, inner token 0..63
constexpr uint32_t SM_RM_LO = SM_RM + 16384;
constexpr uint32_t SM_STG = SM_RM_LO + 16384; // staged chunk rows: q bf16 [64][128], k bf16, log_alpha fp32
constexpr uint32_t SM_STG_K = SM_STG + 16384;
constexpr uint32_t SM_STG_A = SM_STG + 32768;
constexpr uint32_t SM_E = SM_STG + 65536;     // E, then Delta - E: outer token, inner column 0..31
constexpr uint32_t SM_E_LO = SM_E + 4096;
constexpr uint32_t SM_D = SM_E_LO + 4096;     // Delta
constexpr uint32_t SM_D_LO = SM_D + 4096;
constexpr uint32_t SM_BETA = SM_D_LO + 4096;  // fp32 [64]
constexpr uint32_t SM_EM = SM_BETA + 256;     // fp32 [128] e^{m}
constexpr uint32_t SM_GAM = SM_EM + 512;      // fp32 [128] e^{G_last}
constexpr uint32_t SM_EL = SM_GAM + 512;      // fp32 [128] e^{G_last - m}
constexpr uint32_t SM_MBAR = SM_EL + 512;     // two mbarriers: MMA completion, staged loads
constexpr uint32_t SM_TMEMP = SM_MBAR + 16;   // tensor-memory base address
constexpr uint32_t SM_TOTAL = SM_TMEMP + 16;
static_assert(SM_TOTAL <= 232448, "shared memory");
// After the first product the [Kr; Qr] region is free: it holds the solve's fp32
// A and T ([64][68] each, 16-byte aligned rows) and the token path's scratch.
// The pass-1 exchange (fp32 [3][2][128]) uses the [R; M] region, free until then.
constexpr int kPitch = 68;
constexpr uint32_t SM_AMAT = SM_P, SM_TMAT = SM_P + 64 * kPitch * 4;

// tile strides (bytes): s_outer, s_inner
constexpr uint32_t P_SO = 2048, P_SI = 128;
constexpr uint32_t B_SO = (kNB / 8) * 128, B_SI = 128;
constexpr uint32_t H_SO = 1024, H_SI = 128;
constexpr uint32_t S_SO = 512, S_SI = 128;

// tensor-memory columns
constexpr uint32_t TM_D = 0, TM_D3 = 96, TM_D2 = 128, TM_COLS = 256;

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
    float *sEm = reinterpret_cast<float *>(smem + SM_EM);
    float *sGam = reinterpret_cast<float *>(smem + SM_GAM);
    float *sEl = reinterpret_cast<float *>(smem + SM_EL);
    const __nv_bfloat16 *stq = reinterpret_cast<const __nv_bfloat16 *>(smem + SM_STG);
    const __nv_bfloat16 *stk = reinterpret_cast<const __nv_bfloat16 *>(smem + SM_STG_K);
    const float *sta = reinterpret_cast<const float *>(smem + SM_STG_A);
    const uint32_t mbar = sbase + SM_MBAR, mbar_ld = sbase + SM_MBAR + 8;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int slice = blockIdx.x % kNSL;
    const int bh = blockIdx.x / kNSL;
    const int b = bh / H, h = bh % H;
    const int col0 = slice * kDVS;
    const int lrow = 32 * (warp & 3) + lane;     // tensor-memory lane this thread reads
    const int half = warp >> 2;                  // which half of the columns it reads
    const int ch = tid & (kDK - 1);              // key channel of the per-channel passes
    const int th = tid >> 7;                     // token half (0: 0..31, 1: 32..63) of those passes
    const int nchunks = (T + kC - 1) / kC;
    bool ld_pending = false;                     // a staged copy is armed and not yet waited for

    auto row_q = [&](int chunk, int t) { return (((size_t)b * T + (size_t)chunk * kC + t) * H + h); };

    // ---- stage chunk `chunk`'s q, k, log_alpha rows (thread 0 arms the barrier)
    auto issue_stage = [&](int chunk) {
        const int cc = min(kC, T - chunk * kC);
        ld_pending = true;
        if (tid == 0) mbar_expect_tx(mbar_ld, (uint32_t)cc * 1024u);
        __syncthreads();
        if (tid < 3 * cc) {
            const int which = tid / cc, t = tid % cc;
            const size_t r = row_q(chunk, t);
            if (which == 0) bulk_g2s(sbase + SM_STG + t * 256, q + r * kDK, 256, mbar_ld);
            else if (which == 1) bulk_g2s(sbase + SM_STG_K + t * 256, k + r * kDK, 256, mbar_ld);
            else bulk_g2s(sbase + SM_STG_A + t * 512, log_alpha + r * kDK, 512, mbar_ld);
        }
    };
    // value slice (threads of rows 0..63: 16 columns each) and beta go through registers
    auto load_vb = [&](int chunk, uint4 (&vr)[2], float &br) {
        const int cc = min(kC, T - chunk * kC);
        vr[0] = vr[1] = make_uint4(0u, 0u, 0u, 0u);
        if (lrow < cc) {
            const uint4 *src = reinterpret_cast<const uint4 *>(v + row_q(chunk, lrow) * kDV + col0 + 16 * half);
            vr[0] = src[0];
            vr[1] = src[1];
        }
        br = (tid < cc) ? beta[row_q(chunk, tid)] : 0.f;
    };

    // ---- tensor memory and barriers
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     :: "r"(sbase + SM_TMEMP), "r"(TM_COLS) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (tid == 0) {
        mbar_init(mbar, 1);
        mbar_init(mbar_ld, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + SM_TMEMP);
    const uint32_t tlane = (uint32_t)(32 * (warp & 3)) << 16;
    uint32_t phase = 0, ld_phase = 0;
    bool failed = false;

    // ---- state slice: thread holds row lrow, columns 16*half .. +15
    float S[16];
#pragma unroll
    for (int j = 0; j < 16; ++j)
        S[j] = s0 ? s0[((size_t)bh * kDK + lrow) * kDV + col0 + 16 * half + j] : 0.f;

    uint4 vreg[2];
    float breg;
    if (nchunks > 0) {
        issue_stage(0);
        load_vb(0, vreg, breg);
    }

    for (int n = 0; n < nchunks && !failed; ++n) {
        const int t0 = n * kC;
        const int c = min(kC, T - t0);
        auto gv = [&](int t) { return row_q(n, t) * kDV + col0; };

        // ---- the staged rows of this chunk and beta
        failed = __syncthreads_or(!mbar_wait(mbar_ld, ld_phase)) != 0;
        if (failed) break;
        ld_phase ^= 1;
        ld_pending = false;
        if (tid < kC) sBeta[tid] = breg;

        // ---- pass 1 (two threads per key channel, fp32): log-decay sums and range
        float *xch = reinterpret_cast<float *>(smem + SM_RM);   // [3][2][128]
        {
            float la_r[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) la_r[i] = (32 * th + i < c) ? sta[(32 * th + i) * kDK + ch] : 0.f;
            float run = 0.f, lo = INFINITY, hi = -INFINITY;
            if (32 * th < c) {
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    run += la_r[i];
                    lo = fminf(lo, run);
                    hi = fmaxf(hi, run);
                }
            }
            xch[th * kDK + ch] = run;
            xch[256 + th * kDK + ch] = lo;
            xch[512 + th * kDK + ch] = hi;
        }
        __syncthreads();
        float g_start, g_mid;
        bool wide;
        {
            const float tot0 = xch[ch], tot1 = xch[kDK + ch];
            const float lo = fminf(xch[256 + ch], tot0 + xch[256 + kDK + ch]);
            const float hi = fmaxf(xch[512 + ch], tot0 + xch[512 + kDK + ch]);
            const float gl = tot0 + tot1;
            g_mid = 0.5f * (lo + hi);
            g_start = th ? tot0 : 0.f;
            wide = !(0.5f * (hi - lo) <= kGMaxTc && fabsf(hi) <= 2.f * kGMaxTc && fabsf(lo) <= 2.f * kGMaxTc);
            if (th == 0) {
                sEm[ch] = __expf(g_mid);
                sGam[ch] = __expf(gl);
                sEl[ch] = __expf(gl - g_mid);
            }
        }
        const bool token_path = __syncthreads_or(wide) != 0;

        if (!token_path) {
            // ---- pass 2: Kr, Qr (rows t and 64+t of SM_P), Kb and S' (SM_B)
            {
                float run = g_start;
#pragma unroll 1
                for (int g = 0; g < 4; ++g) {
                    float kr[8], qr[8], kb[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int t = 32 * th + 8 * g + e;
                        float kk = 0.f, qq = 0.f;
                        if (t < c) {
                            run += sta[t * kDK + ch];
                            kk = __bfloat162float(stk[t * kDK + ch]);
                            qq = __bfloat162float(stq[t * kDK + ch]);
                        }
                        const float x = run - g_mid;
                        const float up = __expf(x), dn = __expf(-x);
                        kr[e] = kk * up; qr[e] = scale * qq * up; kb[e] = kk * dn;
                    }
                    const int t8 = 32 * th + 8 * g;
                    const uint32_t o1 = core_off(ch, t8, P_SO, P_SI);
                    const uint32_t o2 = core_off(ch, 64 + t8, P_SO, P_SI);
                    const uint32_t o3 = core_off(ch, t8, B_SO, B_SI);
                    st_split8(smem, SM_P + o1, SM_P_LO + o1, kr);
                    st_split8(smem, SM_P + o2, SM_P_LO + o2, qr);
                    st_split8(smem, SM_B + o3, SM_B_LO + o3, kb);
                }
                const float em = sEm[lrow];
#pragma unroll
                for (int g = 0; g < 2; ++g) {
                    float x[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) x[e] = em * S[8 * g + e];
                    const uint32_t off = core_off(lrow, 64 + 16 * half + 8 * g, B_SO, B_SI);
                    st_split8(smem, SM_B + off, SM_B_LO + off, x);
                }
            }
            proxy_fence();
            __syncthreads();
            if (tid == 0) {
                tc_fence_after();
                // D = [Kr; Qr] [Kb | S']
                mma_split(tmem + TM_D, sbase + SM_P, sbase + SM_P_LO, P_SO, P_SI,
                          sbase + SM_B, sbase + SM_B_LO, B_SO, B_SI, kDK / 16,
                          idesc_bf16(128, kNB, 1, 1), false);
                umma_commit(mbar);
            }
            // the staging area is free: prefetch the next chunk's rows
            if (n + 1 < nchunks) issue_stage(n + 1);
            failed = __syncthreads_or(!mbar_wait(mbar, phase)) != 0;
            phase ^= 1;
            if (failed) break;
            tc_fence_after();

            // ---- A (fp32) and E = V - K~S (rows 0..63); M into [R; M] (rows 64..127)
            float e_reg[16];
            {
                float x[32];
                tmem_ld16(tmem + tlane + TM_D + 32 * half, *reinterpret_cast<float (*)[16]>(x));
                tmem_ld16(tmem + tlane + TM_D + 32 * half + 16, *reinterpret_cast<float (*)[16]>(x + 16));
                if (lrow < 64) {
                    const int i = lrow;
                    float *Am = reinterpret_cast<float *>(smem + SM_AMAT) + i * kPitch;
                    const float bi = sBeta[i];
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const int j = 32 * half + e;
                        Am[j] = (j < i) ? bi * x[e] : 0.f;
                    }
                    float ks[16];
                    tmem_ld16(tmem + tlane + TM_D + 64 + 16 * half, ks);
                    const __nv_bfloat16 *vb = reinterpret_cast<const __nv_bfloat16 *>(vreg);
#pragma unroll
                    for (int e = 0; e < 16; ++e) e_reg[e] = __bfloat162float(vb[e]) - ks[e];
#pragma unroll
                    for (int g = 0; g < 2; ++g) {
                        float y[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) y[e] = e_reg[8 * g + e];
                        const uint32_t o = core_off(i, 16 * half + 8 * g, S_SO, S_SI);
                        st_split8(smem, SM_E + o, SM_E_LO + o, y);
                    }
                } else {
                    const int i = lrow - 64;
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        float y[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int j = 32 * half + 8 * g + e;
                            y[e] = (j <= i) ? x[8 * g + e] : 0.f;
                        }
                        const uint32_t o = core_off(lrow, 32 * half + 8 * g, H_SO, H_SI);
                        st_split8(smem, SM_RM + o, SM_RM_LO + o, y);
                    }
                }
            }
            __syncthreads();

            // ---- T = (I + A)^-1 by recursive doubling 16 -> 32 -> 64, fp32
            {
                float *Am = reinterpret_cast<float *>(smem + SM_AMAT);
                float *Tm = reinterpret_cast<float *>(smem + SM_TMAT);
                if (tid < 64) {
                    // 16 x 16 diagonal blocks by forward substitution, one column per thread
                    // (x_l = 0 for l < j, so every term can be summed unconditionally and
                    // the A loads hoisted ahead of the dependent chain)
                    const int blk = tid >> 4, j = tid & 15, o = 16 * blk;
                    float x[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        float s = (i == j) ? 1.f : 0.f;
#pragma unroll
                        for (int l = 0; l < i; ++l) s -= Am[(o + i) * kPitch + o + l] * x[l];
                        x[i] = s;
                    }
#pragma unroll
                    for (int i = 0; i < 16; ++i) Tm[(o + i) * kPitch + o + j] = x[i];
                } else {
                    // the six strictly-upper 16 x 16 blocks of T are zero
                    for (int e = tid - 64; e < 6 * 256; e += kNT - 64) {
                        const int blk = e >> 8, i = (e >> 4) & 15, j = e & 15;
                        const int rb = (blk < 3) ? 0 : (blk < 5 ? 1 : 2);
                        const int cb = (blk < 3) ? blk + 1 : (blk < 5 ? blk - 1 : 3);
                        Tm[(16 * rb + i) * kPitch + 16 * cb + j] = 0.f;
                    }
                }
                __syncthreads();
                // 16 -> 32: T_ab = -T_aa (A_ab T_bb) for (a, b) = (1, 0), (3, 2)
                const int p = tid >> 6, i16 = (tid >> 2) & 15, jq = tid & 3;
                if (tid < 128) {
                    const int a = 2 * p + 1, bb = 2 * p;
                    float4 y = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                    for (int l = 0; l < 16; ++l) {
                        const float av = Am[(16 * a + i16) * kPitch + 16 * bb + l];
                        const float4 tv = *reinterpret_cast<const float4 *>(Tm + (16 * bb + l) * kPitch + 16 * bb + 4 * jq);
                        y.x += av * tv.x; y.y += av * tv.y; y.z += av * tv.z; y.w += av * tv.w;
                    }
                    *reinterpret_cast<float4 *>(Am + (16 * bb + i16) * kPitch + 16 * a + 4 * jq) = y;
                }
                __syncthreads();
                if (tid < 128) {
                    const int a = 2 * p + 1, bb = 2 * p;
                    float4 y = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                    for (int l = 0; l < 16; ++l) {
                        const float tv = Tm[(16 * a + i16) * kPitch + 16 * a + l];
                        const float4 yv = *reinterpret_cast<const float4 *>(Am + (16 * bb + l) * kPitch + 16 * a + 4 * jq);
                        y.x += tv * yv.x; y.y += tv * yv.y; y.z += tv * yv.z; y.w += tv * yv.w;
                    }
                    *reinterpret_cast<float4 *>(Tm + (16 * a + i16) * kPitch + 16 * bb + 4 * jq) =
                        make_float4(-y.x, -y.y, -y.z, -y.w);
                }
                __syncthreads();
                // 32 -> 64: T[32:64, 0:32] = -T[32:64, 32:64] (A[32:64, 0:32] T[0:32, 0:32])
                const int i32 = tid >> 3, jq8 = tid & 7;
                {
                    float4 y = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
                    for (int l = 0; l < 32; ++l) {
                        const float av = Am[(32 + i32) * kPitch + l];
                        const float4 tv = *reinterpret_cast<const float4 *>(Tm + l * kPitch + 4 * jq8);
                        y.x += av * tv.x; y.y += av * tv.y; y.z += av * tv.z; y.w += av * tv.w;
                    }
                    *reinterpret_cast<float4 *>(Am + i32 * kPitch + 32 + 4 * jq8) = y;
                }
                __syncthreads();
                {
                    float4 y = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
                    for (int l = 0; l < 32; ++l) {
                        const float tv = Tm[(32 + i32) * kPitch + 32 + l];
                        const float4 yv = *reinterpret_cast<const float4 *>(Am + l * kPitch + 32 + 4 * jq8);
                        y.x += tv * yv.x; y.y += tv * yv.y; y.z += tv * yv.z; y.w += tv * yv.w;
                    }
                    *reinterpret_cast<float4 *>(Tm + (32 + i32) * kPitch + 4 * jq8) =
                        make_float4(-y.x, -y.y, -y.z, -y.w);
                }
                __syncthreads();
                // R = T Diag(beta) into rows 0..63 of [R; M]
                for (int id = tid; id < 512; id += kNT) {
                    const int i = id >> 3, jg = id & 7;
                    const float4 t0v = *reinterpret_cast<const float4 *>(Tm + i * kPitch + 8 * jg);
                    const float4 t1v = *reinterpret_cast<const float4 *>(Tm + i * kPitch + 8 * jg + 4);
                    const float *bj = sBeta + 8 * jg;
                    float y[8] = {t0v.x * bj[0], t0v.y * bj[1], t0v.z * bj[2], t0v.w * bj[3],
                                  t1v.x * bj[4], t1v.y * bj[5], t1v.z * bj[6], t1v.w * bj[7]};
                    const uint32_t o = core_off(i, 8 * jg, H_SO, H_SI);
                    st_split8(smem, SM_RM + o, SM_RM_LO + o, y);
                }
            }
            // the value slice and beta of the next chunk (this chunk's are consumed)
            if (n + 1 < nchunks) load_vb(n + 1, vreg, breg);
            proxy_fence();
            tc_fence_before();
            __syncthreads();
            if (tid == 0) {
                tc_fence_after();
                // D3 = [R; M] E
                mma_split(tmem + TM_D3, sbase + SM_RM, sbase + SM_RM_LO, H_SI, H_SO,
                          sbase + SM_E, sbase + SM_E_LO, S_SO, S_SI, kC / 16,
                          idesc_bf16(128, kDVS, 0, 1), false);
                umma_commit(mbar);
            }
            failed = __syncthreads_or(!mbar_wait(mbar, phase)) != 0;
            phase ^= 1;
            if (failed) break;
            tc_fence_after();

            // ---- Delta = rows 0..63 of D3, and Delta - E, as B operands
            if (lrow < 64) {
                float x[16];
                tmem_ld16(tmem + tlane + TM_D3 + 16 * half, x);
#pragma unroll
                for (int g = 0; g < 2; ++g) {
                    float d[8], de[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        d[e] = x[8 * g + e];
                        de[e] = d[e] - e_reg[8 * g + e];
                    }
                    const uint32_t o = core_off(lrow, 16 * half + 8 * g, S_SO, S_SI);
                    st_split8(smem, SM_D + o, SM_D_LO + o, d);
                    st_split8(smem, SM_E + o, SM_E_LO + o, de);
                }
            }
            proxy_fence();
            tc_fence_before();
            __syncthreads();
            if (tid == 0) {
                tc_fence_after();
                // D2 = Kb^T Delta (Kb read K-major from SM_B);  D3 += [R; M] (Delta - E)
                mma_split(tmem + TM_D2, sbase + SM_B, sbase + SM_B_LO, B_SI, B_SO,
                          sbase + SM_D, sbase + SM_D_LO, S_SO, S_SI, kC / 16,
                          idesc_bf16(128, kDVS, 0, 1), false);
                mma_split(tmem + TM_D3, sbase + SM_RM, sbase + SM_RM_LO, H_SI, H_SO,
                          sbase + SM_E, sbase + SM_E_LO, S_SO, S_SI, kC / 16,
                          idesc_bf16(128, kDVS, 0, 1), true);
                umma_commit(mbar);
            }
            failed = __syncthreads_or(!mbar_wait(mbar, phase)) != 0;
            phase ^= 1;
            if (failed) break;
            tc_fence_after();

            // ---- state update and outputs (O = Q~S + M Delta, rows 64..127)
            {
                float x[16];
                tmem_ld16(tmem + tlane + TM_D2 + 16 * half, x);
                const float gm = sGam[lrow], el = sEl[lrow];
#pragma unroll
                for (int j = 0; j < 16; ++j) S[j] = gm * S[j] + el * x[j];
                if (lrow >= 64) {
                    const int t = lrow - 64;
                    float o1[16], o2[16];
                    tmem_ld16(tmem + tlane + TM_D + 64 + 16 * half, o1);
                    tmem_ld16(tmem + tlane + TM_D3 + 16 * half, o2);
                    if (t < c) {
                        float4 *dst = reinterpret_cast<float4 *>(out + gv(t) + 16 * half);
#pragma unroll
                        for (int g = 0; g < 4; ++g)
                            dst[g] = make_float4(o1[4 * g] + o2[4 * g], o1[4 * g + 1] + o2[4 * g + 1],
                                                 o1[4 * g + 2] + o2[4 * g + 2], o1[4 * g + 3] + o2[4 * g + 3]);
                    }
                }
            }
            tc_fence_before();
        } else {
            // ---- exact token-by-token path for a chunk with a very wide decay range
            float *fS = reinterpret_cast<float *>(smem + SM_P);      // [128][33]
            float *red = fS + kDK * 33;                               // [2][8][32]
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
                    const int cr = rg * RPT + r;
                    sreg[r] *= expf(sta[t * kDK + cr]);
                    pk += sreg[r] * __bfloat162float(stk[t * kDK + cr]);
                }
                red[rg * kDVS + x] = pk;
                __syncthreads();
                float p = 0.f;
#pragma unroll
                for (int j = 0; j < RG; ++j) p += red[j * kDVS + x];
                const float d = sBeta[t] * (__bfloat162float(v[gv(t) + x]) - p);
                float pq = 0.f;
#pragma unroll
                for (int r = 0; r < RPT; ++r) {
                    const int cr = rg * RPT + r;
                    sreg[r] += __bfloat162float(stk[t * kDK + cr]) * d;
                    pq += sreg[r] * __bfloat162float(stq[t * kDK + cr]);
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
            proxy_fence();
            if (n + 1 < nchunks) {
                issue_stage(n + 1);
                load_vb(n + 1, vreg, breg);
            }
        }
        proxy_fence();
        __syncthreads();
    }

    if (failed) {
        // a bounded wait gave up: let any staged copy still in flight land before
        // this CTA's shared memory is released (itself bounded), then report
        if (ld_pending) mbar_wait(mbar_ld, ld_phase);
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
