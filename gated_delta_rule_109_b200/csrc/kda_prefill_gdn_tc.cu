// Chunked prefill of the scalar-gate members of the family -- Gated DeltaNet (one
// decay per token and head) and DeltaNet (no decay) -- on the sm_100a tensor
// cores, bf16 inputs, dk = dv = 128, fp32 state and outputs.
//
// Same token step as KDA with Diag(alpha_t) replaced by the scalar alpha_t
// ("Kimi Delta Attention: The Linear Attention Behind Kimi K2 and Qwen3",
// §DeltaNet, Gated DeltaNet, and KDA: comparison table and FAQ "What's the
// concrete difference between Gated DeltaNet and KDA?"; the DeltaNet update of
// "KDA Technical Deep Dive", §From attention to recurrent state).  With a
// scalar gate the decay leaves every contraction: per chunk of c <= 64 tokens,
// g_t = log alpha_t, G_t = in-chunk inclusive sum, D_ij = e^{G_i - G_j} (<= 1 for
// j <= i when alpha <= 1):
//
//   D_KK = [K ; Q] K^T,   D_S = [K ; Q] S          ([K ; Q] are the exact bf16 inputs)
//   A    = Diag(beta) strictly_lower(D_KK[0:64] (.) D),  M = scale lower(D_KK[64:128] (.) D)
//   T    = (I + A)^-1,  R = T Diag(beta)
//   E    = V - Diag(e^G) D_S[0:64],   Delta = R E
//   O    = scale Diag(e^G) D_S[64:128] + M Delta,   M Delta = M E + M (Delta - E)
//   S   <- e^{G_last} S + K^T Diag(e^{G_last - G}) Delta
//
// Exact operands need no split: K K^T and K Q^T take one tensor-core term, the
// products with S or Delta two (hi and lo of the fp32 side), the products of two
// fp32 operands three.  No exponential is ever larger than 1, so there is no
// wide-range fallback.  Layout and roles as in the per-channel kernel: one CTA
// per (b, h, 32-column value slice), state slice in registers, q and k rows
// staged one chunk ahead by cp.async.bulk and rearranged into the canonical
// operand layout in shared memory.
#include "kda_tc_ptx.cuh"

namespace kda {

__device__ unsigned int g_gdn_device_status;   // bit 0: a bounded wait gave up

namespace {

using namespace tcx;

constexpr int kC = 64, kDK = 128, kDV = 128, kDVS = 32, kNSL = kDV / kDVS, kNT = 256;
constexpr int kPitch = 68;

// ---------------------------------------------------------------- shared memory map
constexpr uint32_t SM_KQ = 0;                  // [K; Q] exact bf16, K-major: outer row 0..127, inner dk
constexpr uint32_t SM_STG = 32768;             // staged rows: q bf16 [64][128], k bf16 [64][128]
constexpr uint32_t SM_STG_K = SM_STG + 16384;
constexpr uint32_t SM_SOL = SM_STG + 32768;    // solve: fp32 A and T, [64][68] each
constexpr uint32_t SM_AMAT = SM_SOL, SM_TMAT = SM_SOL + 64 * kPitch * 4;
constexpr uint32_t SM_S = SM_SOL + 2 * 64 * kPitch * 4;   // S: outer dk, inner column 0..31
constexpr uint32_t SM_S_LO = SM_S + 8192;
constexpr uint32_t SM_RM = SM_S + 16384;       // [R; M]: outer row 0..127, inner token 0..63
constexpr uint32_t SM_RM_LO = SM_RM + 16384;
constexpr uint32_t SM_E = SM_RM + 32768;       // E, then Delta - E: outer token, inner column
constexpr uint32_t SM_E_LO = SM_E + 4096;
constexpr uint32_t SM_D = SM_E + 8192;         // e^{G_last - G} Delta
constexpr uint32_t SM_D_LO = SM_D + 4096;
constexpr uint32_t SM_SC = SM_D + 8192;        // fp32 [4][64]: beta, G, e^G, e^{G_last - G}
constexpr uint32_t SM_MBAR = SM_SC + 4 * 256;  // mbarriers: MMA completion, staged loads
constexpr uint32_t SM_TMEMP = SM_MBAR + 16;
constexpr uint32_t SM_TOTAL = SM_TMEMP + 16;
static_assert(SM_TOTAL <= 232448, "shared memory");

constexpr uint32_t KQ_SO = 2048, KQ_SI = 128;  // K-major 128 x 128
constexpr uint32_t H_SO = 1024, H_SI = 128;    // K-major 128 x 64
constexpr uint32_t S_SO = 512, S_SI = 128;     // MN-major 128 x 32 / 64 x 32

constexpr uint32_t TM_KK = 0, TM_DS = 64, TM_D3 = 96, TM_D2 = 128, TM_COLS = 256;

__global__ void __launch_bounds__(kNT, 1)
prefill_gdn_tc_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                      const __nv_bfloat16 *__restrict__ v, const float *__restrict__ log_alpha,
                      const float *__restrict__ beta, const float *__restrict__ s0,
                      float *__restrict__ out, float *__restrict__ sT, int T, int H, float scale)
{
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t sbase = (uint32_t)__cvta_generic_to_shared(smem);
    float *sBeta = reinterpret_cast<float *>(smem + SM_SC);
    float *sG = sBeta + 64;
    float *sEg = sBeta + 128;
    float *sEl = sBeta + 192;
    const uint32_t mbar = sbase + SM_MBAR, mbar_ld = mbar + 8;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int slice = blockIdx.x % kNSL;
    const int bh = blockIdx.x / kNSL;
    const int b = bh / H, h = bh % H;
    const int col0 = slice * kDVS;
    const int lrow = 32 * (warp & 3) + lane;
    const int half = warp >> 2;
    const int nchunks = (T + kC - 1) / kC;
    bool ld_pending = false;

    auto row_q = [&](int chunk, int t) { return (((size_t)b * T + (size_t)chunk * kC + t) * H + h); };
    auto chunk_len = [&](int chunk) { return min(kC, T - chunk * kC); };

    auto issue_stage = [&](int chunk) {
        const int cc = chunk_len(chunk);
        ld_pending = true;
        if (tid == 0) mbar_expect_tx(mbar_ld, (uint32_t)cc * 512u);
        __syncthreads();
        if (tid < 2 * cc) {
            const int t = tid % cc;
            const size_t r = row_q(chunk, t);
            if (tid < cc) bulk_g2s(sbase + SM_STG + t * 256, q + r * kDK, 256, mbar_ld);
            else bulk_g2s(sbase + SM_STG_K + t * 256, k + r * kDK, 256, mbar_ld);
        }
    };
    // per-token scalars (beta, log alpha; threads 0..63) and the value slice (rows 0..63)
    auto load_tok = [&](int chunk, uint4 (&vr)[2], float &br, float &gr) {
        const int cc = chunk_len(chunk);
        vr[0] = vr[1] = make_uint4(0u, 0u, 0u, 0u);
        if (lrow < cc) {
            const uint4 *src = reinterpret_cast<const uint4 *>(v + row_q(chunk, lrow) * kDV + col0 + 16 * half);
            vr[0] = src[0];
            vr[1] = src[1];
        }
        br = (tid < cc) ? beta[row_q(chunk, tid)] : 0.f;
        gr = (tid < cc && log_alpha) ? log_alpha[row_q(chunk, tid)] : 0.f;
    };

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
    auto wait_mma = [&]() -> bool {
        const bool bad = (tid == 0) && !mbar_wait(mbar, phase);
        phase ^= 1;
        return __syncthreads_or(bad) != 0;
    };

    float S[16];
#pragma unroll
    for (int j = 0; j < 16; ++j)
        S[j] = s0 ? s0[((size_t)bh * kDK + lrow) * kDV + col0 + 16 * half + j] : 0.f;

    uint4 vreg[2];
    float breg = 0.f, greg = 0.f;
    if (nchunks > 0) {
        issue_stage(0);
        load_tok(0, vreg, breg, greg);
    }

    for (int n = 0; n < nchunks && !failed; ++n) {
        const int c = chunk_len(n);

        // ---- staged rows -> [K; Q] operand; the chunk's scalars; S as a split B operand
        failed = __syncthreads_or(tid == 0 && !mbar_wait(mbar_ld, ld_phase)) != 0;
        if (failed) break;
        ld_phase ^= 1;
        ld_pending = false;
        for (int id = tid; id < 2 * 64 * 16; id += kNT) {
            const int which = id >> 10, t = (id >> 4) & 63, kb = id & 15;
            uint4 val = make_uint4(0u, 0u, 0u, 0u);
            if (t < c) val = *reinterpret_cast<const uint4 *>(smem + (which ? SM_STG : SM_STG_K) + t * 256 + kb * 16);
            *reinterpret_cast<uint4 *>(smem + SM_KQ + core_off(which * 64 + t, 8 * kb, KQ_SO, KQ_SI)) = val;
        }
        if (warp < 2) {
            // inclusive scan of log alpha over the chunk (two warps of 32 tokens)
            float gsum = greg;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float up = __shfl_up_sync(0xffffffffu, gsum, o);
                if (lane >= o) gsum += up;
            }
            sG[tid] = gsum;
            sBeta[tid] = breg;
        }
#pragma unroll
        for (int g = 0; g < 2; ++g) {
            float xv[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) xv[e] = S[8 * g + e];
            const uint32_t off = core_off(lrow, 16 * half + 8 * g, S_SO, S_SI);
            st_split8(smem, SM_S + off, SM_S_LO + off, xv);
        }
        __syncthreads();
        float gt = 0.f, glast = 0.f;
        if (tid < 64) {
            gt = sG[tid] + ((tid >= 32) ? sG[31] : 0.f);   // the two warps' scans joined
            glast = sG[31] + sG[63];
        }
        __syncthreads();
        if (tid < 64) {
            sG[tid] = gt;
            sEg[tid] = __expf(gt);
            sEl[tid] = __expf(glast - gt);
        }
        proxy_fence();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            // D_KK = [K; Q] K^T (exact operands: one term); D_S = [K; Q] S (two terms)
            mma_split(tmem + TM_KK, sbase + SM_KQ, 0u, KQ_SI, KQ_SO, sbase + SM_KQ, 0u, KQ_SI, KQ_SO,
                      kDK / 16, idesc_bf16(128, 64, 0, 0), false, false, false);
            mma_split(tmem + TM_DS, sbase + SM_KQ, 0u, KQ_SI, KQ_SO, sbase + SM_S, sbase + SM_S_LO, S_SO, S_SI,
                      kDK / 16, idesc_bf16(128, kDVS, 0, 1), false, false, true);
            umma_commit(mbar);
        }
        // the staging area is free: prefetch the next chunk's rows
        if (n + 1 < nchunks) issue_stage(n + 1);
        failed = wait_mma();
        if (failed) break;
        tc_fence_after();

        // ---- A (fp32) and E = V - e^G D_S (rows 0..63); M into [R; M] (rows 64..127)
        float e_reg[16];
        {
            float x[32];
            tmem_ld16(tmem + tlane + TM_KK + 32 * half, *reinterpret_cast<float (*)[16]>(x));
            tmem_ld16(tmem + tlane + TM_KK + 32 * half + 16, *reinterpret_cast<float (*)[16]>(x + 16));
            const int i = lrow & 63;
            const float gi = sG[i];
            if (lrow < 64) {
                float *Am = reinterpret_cast<float *>(smem + SM_AMAT) + i * kPitch;
                const float bi = sBeta[i];
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int j = 32 * half + e;
                    Am[j] = (j < i) ? bi * x[e] * __expf(gi - sG[j]) : 0.f;
                }
                float ks[16];
                tmem_ld16(tmem + tlane + TM_DS + 16 * half, ks);
                const float eg = sEg[i];
                const __nv_bfloat16 *vb = reinterpret_cast<const __nv_bfloat16 *>(vreg);
#pragma unroll
                for (int e = 0; e < 16; ++e) e_reg[e] = __bfloat162float(vb[e]) - eg * ks[e];
#pragma unroll
                for (int g = 0; g < 2; ++g) {
                    float y[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) y[e] = e_reg[8 * g + e];
                    const uint32_t o = core_off(i, 16 * half + 8 * g, S_SO, S_SI);
                    st_split8(smem, SM_E + o, SM_E_LO + o, y);
                }
            } else {
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    float y[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int j = 32 * half + 8 * g + e;
                        y[e] = (j <= i) ? scale * x[8 * g + e] * __expf(gi - sG[j]) : 0.f;
                    }
                    const uint32_t o = core_off(lrow, 32 * half + 8 * g, H_SO, H_SI);
                    st_split8(smem, SM_RM + o, SM_RM_LO + o, y);
                }
            }
        }
        if (n + 1 < nchunks) load_tok(n + 1, vreg, breg, greg);
        __syncthreads();

        // ---- T = (I + A)^-1 by recursive doubling 16 -> 32 -> 64, fp32; R = T Diag(beta)
        {
            float *Am = reinterpret_cast<float *>(smem + SM_AMAT);
            float *Tm = reinterpret_cast<float *>(smem + SM_TMAT);
            if (tid < 64) {
                const int blk = tid >> 4, j = tid & 15, o = 16 * blk;
                float xs[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    float s = (i == j) ? 1.f : 0.f;
#pragma unroll
                    for (int l = 0; l < i; ++l) s -= Am[(o + i) * kPitch + o + l] * xs[l];
                    xs[i] = s;
                }
#pragma unroll
                for (int i = 0; i < 16; ++i) Tm[(o + i) * kPitch + o + j] = xs[i];
            } else {
                for (int e = tid - 64; e < 6 * 256; e += kNT - 64) {
                    const int blk = e >> 8, i = (e >> 4) & 15, j = e & 15;
                    const int rb = (blk < 3) ? 0 : (blk < 5 ? 1 : 2);
                    const int cb = (blk < 3) ? blk + 1 : (blk < 5 ? blk - 1 : 3);
                    Tm[(16 * rb + i) * kPitch + 16 * cb + j] = 0.f;
                }
            }
            __syncthreads();
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
        proxy_fence();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            // D3 = [R; M] E
            mma_split(tmem + TM_D3, sbase + SM_RM, sbase + SM_RM_LO, H_SI, H_SO,
                      sbase + SM_E, sbase + SM_E_LO, S_SO, S_SI, kC / 16, idesc_bf16(128, kDVS, 0, 1), false);
            umma_commit(mbar);
        }
        failed = wait_mma();
        if (failed) break;
        tc_fence_after();

        // ---- e^{G_last - G} Delta and Delta - E as B operands
        if (lrow < 64) {
            float x[16];
            tmem_ld16(tmem + tlane + TM_D3 + 16 * half, x);
            const float el = sEl[lrow];
#pragma unroll
            for (int g = 0; g < 2; ++g) {
                float d[8], de[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    d[e] = el * x[8 * g + e];
                    de[e] = x[8 * g + e] - e_reg[8 * g + e];
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
            // D2 = K^T (e^{G_last-G} Delta): K rows of [K; Q] read MN-major (M = dk, K = token);
            // D3 += [R; M] (Delta - E)
            mma_split(tmem + TM_D2, sbase + SM_KQ, 0u, KQ_SO, KQ_SI, sbase + SM_D, sbase + SM_D_LO, S_SO, S_SI,
                      kC / 16, idesc_bf16(128, kDVS, 1, 1), false, false, true);
            mma_split(tmem + TM_D3, sbase + SM_RM, sbase + SM_RM_LO, H_SI, H_SO,
                      sbase + SM_E, sbase + SM_E_LO, S_SO, S_SI, kC / 16, idesc_bf16(128, kDVS, 0, 1), true);
            umma_commit(mbar);
        }
        failed = wait_mma();
        if (failed) break;
        tc_fence_after();

        // ---- state update and outputs
        {
            float x[16];
            tmem_ld16(tmem + tlane + TM_D2 + 16 * half, x);
            const float gl = sEg[63];                       // e^{G_last} (padded rows repeat it)
#pragma unroll
            for (int j = 0; j < 16; ++j) S[j] = gl * S[j] + x[j];
            if (lrow >= 64) {
                const int t = lrow - 64;
                float o1[16], o2[16];
                tmem_ld16(tmem + tlane + TM_DS + 16 * half, o1);
                tmem_ld16(tmem + tlane + TM_D3 + 16 * half, o2);
                if (t < c) {
                    const float sq = scale * sEg[t];
                    float4 *dst = reinterpret_cast<float4 *>(out + row_q(n, t) * kDV + col0 + 16 * half);
#pragma unroll
                    for (int g = 0; g < 4; ++g)
                        dst[g] = make_float4(sq * o1[4 * g] + o2[4 * g], sq * o1[4 * g + 1] + o2[4 * g + 1],
                                             sq * o1[4 * g + 2] + o2[4 * g + 2], sq * o1[4 * g + 3] + o2[4 * g + 3]);
                }
            }
        }
        tc_fence_before();
        proxy_fence();
        __syncthreads();
    }

    if (failed) {
        if (ld_pending) mbar_wait(mbar_ld, ld_phase);
        if (tid == 0) atomicOr(&g_gdn_device_status, 1u);
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

cudaError_t launch_prefill_gdn_tc(const ForwardArgs &a, cudaStream_t stream)
{
    cudaError_t e = cudaFuncSetAttribute(prefill_gdn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SM_TOTAL);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)((size_t)a.B * a.H * kNSL);
    prefill_gdn_tc_kernel<<<grid, kNT, SM_TOTAL, stream>>>(
        static_cast<const __nv_bfloat16 *>(a.q), static_cast<const __nv_bfloat16 *>(a.k),
        static_cast<const __nv_bfloat16 *>(a.v), a.log_alpha, a.beta, a.s0, a.out, a.sT, a.T, a.H,
        a.scale);
    e = cudaGetLastError();
    if (e == cudaSuccess) note_launch();
    return e;
}

cudaError_t take_gdn_device_status(unsigned int *status)
{
    unsigned int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbol(status, g_gdn_device_status, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    if (*status) e = cudaMemcpyToSymbol(g_gdn_device_status, &zero, sizeof(unsigned int));
    return e;
}

}  // namespace kda
