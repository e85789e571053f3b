// Two-kernel chunked KDA prefill on the sm_100a tensor cores, bf16 inputs,
// dk = dv = 128, fp32 state and outputs: the chunk-local work of every chunk
// runs in parallel (prefill_prep_kernel; prefill_prep_scalar_kernel for a scalar
// gate), and only the short state chain runs in sequence (prefill_chain_t_kernel,
// one CTA per (b, h); prefill_chain_kernel, one per (b, h, 32-column slice)).
//
// The token step is the one of "Kimi Delta Attention: The Linear Attention
// Behind Kimi K2 and Qwen3", §How Kimi Delta Attention works step by step; the
// sequence is processed chunkwise with the chunk-boundary state as the next
// chunk's initial condition ("KDA Technical Deep Dive", §Systems and
// implementation tradeoffs, Training).  Per (b, h) and chunk of c <= 64 tokens
// with entering state S, G_t = in-chunk inclusive sum of log_alpha:
//
//   Kr = k e^{G-m},  Qr = scale q e^{G-m},  Kb = k e^{m-G}      (m: per-channel reference point)
//   A = Diag(beta) strictly_lower(Kr Kb^T),  M = lower(Qr Kb^T)
//   R = (I + A)^-1 Diag(beta),  Wr = R Kr,  U = R V
//   S'    = Diag(e^m) S
//   Delta = R (V - (k e^G) S) = U - Wr S'         (row t = the token step's error e_t)
//   O     = Qr S' + M Delta
//   S    <- Diag(e^{G_last}) S + Diag(e^{G_last - m}) Kb^T Delta
//
// Nothing above except S', Delta, O and the update depends on S, so the
// chunk-local kernel computes it for all chunks at once and writes one record per
// chunk to a workspace; a chain kernel then walks the chunks of each (b, h) with two
// tensor-core round trips per chunk:  D1 = [Wr ; Qr] S'  ->  Delta = U - D1[0:64];
// D2 = Kb^T Delta, D3 = M Delta  ->  S update and O = D1[64:128] + D3.  For few heads
// and long sequences the two kernels run side by side on alternating blocks of chunks
// (run_pipelined).
//
// m is the midpoint of the chunk's first and last G, so each split factor is at
// most e^{range/2} for a monotone decay; a chunk where some |G - m| > 40 instead
// computes A and M pair by pair with e^{G_i - G_j} <= 1 and stores k e^G, scale
// q e^G and k e^{G_last - G} in place of Kr, Qr and Kb (with e^m = e^{G_last - m} = 1).
//
// Precision: every derived fp32 operand X is split X = hi + lo (bf16 each) and a
// product takes hi*hi + lo*hi + hi*lo (an exact bf16 input needs no lo part);
// accumulation is fp32 in tensor memory.
//
// Records hold their tiles in the byte order of the no-swizzle canonical
// operand layout (core matrices of 8 rows x 16 bytes), so the chain kernel
// brings them into shared memory with plain cp.async.bulk copies.  Every
// mbarrier wait is bounded; a wait that runs out records KDA_ERR_TIMEOUT in a
// device status word and the CTA stops after its copies in flight have landed.
#include <algorithm>
#include <mutex>
#include <string.h>

#include <cudaTypedefs.h>

#include "kda_tc_ptx.cuh"

namespace kda {

__device__ unsigned int g_split_device_status;   // bit 0: a bounded wait gave up

namespace {

using namespace tcx;

constexpr int kC = 64, kDK = 128, kDV = 128, kDVS = 32, kNSL = kDV / kDVS, kNT = 256;
constexpr float kGMaxTc = 40.f;
constexpr int kPitch = 68;

// ---------------------------------------------------------------- chunk record (bytes)
// [Wr ; Qr]: K-major A tile (outer row 0..127, inner dk), then e^m fp32 [dk]
constexpr uint32_t R_WQ = 0, R_WQ_LO = 32768, R_EM = 65536;
constexpr uint32_t kWqBytes = 65536 + 512;
// Kb read as the MN-major A tile of Kb^T (outer token, inner dk)
constexpr uint32_t R_KT = R_WQ + kWqBytes, R_KT_LO = R_KT + 16384;
// M: rows 64..127 of a K-major A tile (outer row, inner token)
constexpr uint32_t R_M = R_KT + 32768, R_M_LO = R_M + 8192;
// U fp32 [value slice][token][32];  e^{G_last} and e^{G_last - m} fp32 [dk] each
constexpr uint32_t R_U = R_M + 16384, R_GAM = R_U + 32768, R_EL = R_GAM + 512;
constexpr uint32_t kRec = R_EL + 512;
static_assert(kRec % 16 == 0 && R_KT % 16 == 0, "bulk-copy alignment");
// The chunk-local kernels stage U as the 256 rows (slice, token) of 128 bytes of one
// TMA box with the 128-byte swizzle (16-byte piece j of row r at piece j ^ (r % 8)), so
// that the 32 tokens a warp writes at once fall on distinct banks; the tensor store
// writes the record's plain [slice][token][32] order.
__device__ __forceinline__ uint32_t u_stage_off(int r, int j)
{
    return (uint32_t)r * 128u + ((uint32_t)(j ^ (r & 7)) << 4);
}

constexpr uint32_t RW_SO = 2048, RW_SI = 128;   // outer row or token (8 per group), inner dk (128)
constexpr uint32_t H_SO = 1024, H_SI = 128;     // outer row, inner token (64)
constexpr uint32_t S_SO = 512, S_SI = 128;      // outer dk or token (K), inner column (N = 32)

// ---------------------------------------------------------------- prep kernel smem
// Tiles are K-major with outer = token/row and inner = key channel (RW_SO/RW_SI):
// [Kr; Qr] is the A of the first product, Kb its B, and the Kr rows are read
// again (MN-major) as the B of W = R Kr.  Layout chosen so that what is free after
// the first product (Qr, Kb) is contiguous enough for the solve.
constexpr uint32_t PP_P = 0;            // [Kr hi ; Qr hi]  (Kr hi 0..16K, Qr hi 16K..32K)
constexpr uint32_t PP_KB = 32768;       // Kb hi, Kb lo
constexpr uint32_t PP_KB_LO = 49152;
constexpr uint32_t PP_P_LO = 65536;     // [Kr lo ; Qr lo]
constexpr uint32_t PP_V = 98304;        // V: MN-major B (outer token, inner column)
constexpr uint32_t PP_BETA = 114688;    // fp32 [64]
constexpr uint32_t PP_MBAR = PP_BETA + 256;
constexpr uint32_t PP_TMEMP = PP_MBAR + 8;
constexpr uint32_t PP_TOTAL = PP_TMEMP + 8;
static_assert(PP_TOTAL <= 115712, "two CTAs per SM");
// after the first product: fp32 A and T of the solve over Qr hi and Kb; R (K-major,
// outer row, inner token) over Qr lo; a 128-row view of R hi or R lo stays in smem
constexpr uint32_t PP_AMAT = 16384, PP_TMAT = PP_AMAT + 64 * kPitch * 4;
constexpr uint32_t PP_R = 81920, PP_R_LO = PP_R + 8192;
static_assert(PP_TMAT + 64 * kPitch * 4 <= PP_P_LO, "solve scratch");
// wide-range path: G fp32 [64][128] over Qr hi and Kb hi, pairwise A (pitch 64) over Kb lo
constexpr uint32_t PP_G = 16384, PP_AW = 49152;
// the scan: log_alpha transposed through shared memory (row pitch 132 floats keeps the
// 16-byte row accesses of a quarter warp on distinct banks), over Qr hi and Kb before
// the split pass writes them; half totals after the per-channel scalars in the V region
constexpr int kGP = 132;
constexpr uint32_t PP_GS = 16384;
static_assert(PP_GS + 64 * kGP * 4 <= PP_P_LO, "scan scratch");

constexpr uint32_t TMP_AM = 0, TMP_W = 0, TMP_U = 128, TMP_COLS = 256;

// T = (I + A)^-1 for a strictly lower triangular 64 x 64 fp32 A (row pitch kPitch),
// by forward substitution on the four 16 x 16 diagonal blocks and recursive doubling
// 16 -> 32 -> 64 (T21 = -T22 A21 T11 at each level), all in fp32.  Called by every
// thread of a 256-thread CTA; A is overwritten with intermediate products, and T is
// complete (every thread may read it) after the caller's next __syncthreads().
__device__ __forceinline__ void unit_lower_inverse(float *__restrict__ Am, float *__restrict__ Tm, int tid)
{
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
}

__global__ void __launch_bounds__(kNT, 2)
prefill_prep_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                    const __nv_bfloat16 *__restrict__ v, const float *__restrict__ log_alpha,
                    const float *__restrict__ beta, uint8_t *__restrict__ ws, int T, int H,
                    int n0, int nb, float scale, int prep_flags, int gate, int pf_dist,
                    const __grid_constant__ CUtensorMap u_map)
{
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t sbase = (uint32_t)__cvta_generic_to_shared(smem);
    float *sBeta = reinterpret_cast<float *>(smem + PP_BETA);
    const uint32_t mbar = sbase + PP_MBAR;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // CTAs in launch order take the block's chunks from the last to the first, every
    // (b, h) of a chunk together: the chunks the chain reads first are written last and
    // are still in L2 when it starts
    const int nbh = (int)(gridDim.x / (unsigned)nb);
    const int bh = (int)blockIdx.x % nbh;
    const int nloc = nb - 1 - (int)blockIdx.x / nbh;  // chunk within this block
    const int b = bh / H, h = bh % H;
    const int t0 = (n0 + nloc) * kC;
    const int c = min(kC, T - t0);
    const int lrow = 32 * (warp & 3) + lane;          // tensor-memory lane of the readouts
    const int half = warp >> 2;
    const int ch0 = 16 * warp;                        // pass 1/2: channels ch0..ch0+15, tokens lane, lane+32
    const bool gate_act = (prep_flags & kPrepLogsigmoidGate) != 0;   // log_alpha holds gate pre-activations
    const bool norm_qk = (prep_flags & kPrepNormalizeQK) != 0;       // q, k are L2-normalised here
    uint8_t *rec = ws + ((size_t)bh * nb + nloc) * kRec;
    auto row = [&](int t) { return ((size_t)b * T + t0 + t) * H + h; };
    auto la_at = [&](int t, int chn) -> float {
        return gate == KDA_GATE_CHANNEL ? log_alpha[row(t) * kDK + chn]
               : gate == KDA_GATE_SCALAR ? log_alpha[row(t)] : 0.f;
    };

    // ---- loads, all issued at once (one DRAM latency per CTA): log_alpha rows and beta
    // by cp.async into shared memory (rows past the chunk's end zero-filled), the k and
    // q of this thread's four (token, 8 channels) items into registers; V follows by
    // cp.async once the V region has served as scratch
    float *Gs = reinterpret_cast<float *>(smem + PP_GS);
    if (gate == KDA_GATE_CHANNEL) {
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            const int id = tid + kNT * r, t = id >> 5, j = id & 31;
            const bool okt = t < c;
            cp_async16(sbase + PP_GS + (uint32_t)(t * kGP + 4 * j) * 4u, log_alpha + row(okt ? t : 0) * kDK + 4 * j,
                       okt ? 16u : 0u);
        }
    } else {
        // one decay per token and head (Gated DeltaNet) or none (DeltaNet): the
        // token's value repeated over the key channels, so the rest is unchanged
        const int t = tid >> 2, c0 = 32 * (tid & 3);
        const float g = (gate == KDA_GATE_SCALAR && t < c) ? log_alpha[row(t)] : 0.f;
#pragma unroll
        for (int j = 0; j < 32; j += 4)
            *reinterpret_cast<float4 *>(Gs + t * kGP + c0 + j) = make_float4(g, g, g, g);
    }
    if (tid < kC) {
        // beta is [B, T, H]: the chunk's 64 values are H apart, so they come one by one,
        // with the log_alpha rows (zero past the chunk's end)
        const bool okt = tid < c;
        cp_async4(sbase + PP_BETA + 4u * tid, beta + row(okt ? tid : 0), okt ? 4u : 0u);
    }
    uint4 kv4[4], qv4[4];
#pragma unroll
    for (int item = 0; item < 4; ++item) {
        const int t = lane + 32 * (item >> 1);
        const bool okt = t < c;
        const size_t o = row(okt ? t : 0) * kDK + ch0 + 8 * (item & 1);
        kv4[item] = okt ? *reinterpret_cast<const uint4 *>(k + o) : make_uint4(0u, 0u, 0u, 0u);
        qv4[item] = okt ? *reinterpret_cast<const uint4 *>(q + o) : make_uint4(0u, 0u, 0u, 0u);
    }
    cp_async_commit();
    // warm L2 with the inputs of the CTA pf_dist places further on, which starts while
    // this one is still busy: its load phase then reads L2 rather than DRAM
    if (pf_dist > 0 && blockIdx.x + (unsigned)pf_dist < gridDim.x) {
        const int xb = (int)blockIdx.x + pf_dist;
        const int pbh = xb % nbh, pb = pbh / H, ph = pbh % H;
        const int pt0 = (n0 + nb - 1 - xb / nbh) * kC, pc = min(kC, T - pt0);
        const int t = tid >> 2, which = tid & 3;
        if (t < pc) {
            const size_t r = ((size_t)pb * T + pt0 + t) * H + ph;
            if (which == 0) l2_prefetch(q + r * kDK, kDK * 2);
            else if (which == 1) l2_prefetch(k + r * kDK, kDK * 2);
            else if (which == 2) l2_prefetch(v + r * kDV, kDV * 2);
            else {
                if (gate == KDA_GATE_CHANNEL) l2_prefetch(log_alpha + r * kDK, kDK * 4);
                asm volatile("prefetch.global.L2 [%0];" :: "l"(beta + r) : "memory");
            }
        }
    }

    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     :: "r"(sbase + PP_TMEMP), "r"(TMP_COLS) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (tid == 0) {
        mbar_init(mbar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    cp_async_wait_all();
    __syncthreads();

    // ---- in-chunk inclusive sums over tokens, per channel, in shared memory: thread
    // (channel, token half) sums its 32 tokens in order, the second half then adds the
    // first half's total.
    // Padded tokens add 0.  Per channel: G_last (the sum up to the chunk's last token),
    // the reference point m midway between the first and last G (the extremes when the
    // decay is monotone), and the chunk's minimum and maximum of G, which decide whether
    // some split factor e^{|G - m|} could overflow (the same decision as testing every
    // token: G - m rounds monotonically in G).
    float *sGm = reinterpret_cast<float *>(smem + PP_V);
    float *sGl = sGm + kDK;
    float *sTot = sGm + 2 * kDK;
    float *sMin = sGm + 5 * kDK, *sMax = sGm + 7 * kDK;   // [2][128] each, after sInv
    {
        const int ch = tid & (kDK - 1), th = tid >> 7;
        float run = 0.f, lo = 3.0e38f, hi = -3.0e38f;
        if (gate_act) {
#pragma unroll 8
            for (int i = 0; i < 32; ++i) {
                float *gp = Gs + (32 * th + i) * kGP + ch;
                run += (32 * th + i < c) ? log_sigmoid(*gp) : 0.f;
                *gp = run;
                lo = fminf(lo, run);
                hi = fmaxf(hi, run);
            }
        } else {
            // separate loop: no log-sigmoid evaluated (and discarded) per element
#pragma unroll 8
            for (int i = 0; i < 32; ++i) {
                float *gp = Gs + (32 * th + i) * kGP + ch;
                run += *gp;
                *gp = run;
                lo = fminf(lo, run);
                hi = fmaxf(hi, run);
            }
        }
        sTot[th * kDK + ch] = run;
        sMin[th * kDK + ch] = lo;
        sMax[th * kDK + ch] = hi;
    }
    __syncthreads();
    bool wide = false;      // some |G - m| > 40 (or |m| > 80): the split exponentials could overflow
    {
        const int ch = tid & (kDK - 1), th = tid >> 7;
        const float tot0 = sTot[ch];
        if (th == 1) {
#pragma unroll 8
            for (int i = 0; i < 32; ++i) Gs[(32 + i) * kGP + ch] += tot0;
        } else {
            const float g_l = tot0 + sTot[kDK + ch];
            const float g_m = 0.5f * (Gs[ch] + g_l);
            const float gmin = fminf(sMin[ch], sMin[kDK + ch] + tot0);
            const float gmax = fmaxf(sMax[ch], sMax[kDK + ch] + tot0);
            wide = !(gmax - g_m <= kGMaxTc && g_m - gmin <= kGMaxTc && fabsf(g_m) <= 2.f * kGMaxTc);
            sGm[ch] = g_m;
            sGl[ch] = g_l;
            reinterpret_cast<float *>(rec + R_EM)[ch] = __expf(g_m);
            reinterpret_cast<float *>(rec + R_GAM)[ch] = __expf(g_l);
            reinterpret_cast<float *>(rec + R_EL)[ch] = __expf(g_l - g_m);
        }
    }
    const bool wide_path = __syncthreads_or(wide) != 0;
    float G[2][16];
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
        const float4 *src = reinterpret_cast<const float4 *>(Gs + (lane + 32 * hf) * kGP + ch0);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float4 gv = src[j];
            G[hf][4 * j] = gv.x; G[hf][4 * j + 1] = gv.y; G[hf][4 * j + 2] = gv.z; G[hf][4 * j + 3] = gv.w;
        }
    }
    __syncthreads();
    // ---- optional L2 normalisation of q and k rows: squared-norm partials of this
    // thread's 16 channels, summed over the eight warps through the (now free) scratch
    float inv_k[2] = {1.f, 1.f}, inv_q[2] = {1.f, 1.f};
    float *sInv = sGm + 4 * kDK;            // [2][64]: 1/|k_t|, 1/|q_t| (for the wide path)
    if (norm_qk) {
        float *part = Gs;                   // [2][8 warps][64 tokens]
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            float sk = 0.f, sq = 0.f;
#pragma unroll
            for (int g = 0; g < 2; ++g) {
                const __nv_bfloat16 *kb16 = reinterpret_cast<const __nv_bfloat16 *>(&kv4[2 * hf + g]);
                const __nv_bfloat16 *qb16 = reinterpret_cast<const __nv_bfloat16 *>(&qv4[2 * hf + g]);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float kf = __bfloat162float(kb16[i]), qf = __bfloat162float(qb16[i]);
                    sk += kf * kf;
                    sq += qf * qf;
                }
            }
            part[warp * kC + lane + 32 * hf] = sk;
            part[8 * kC + warp * kC + lane + 32 * hf] = sq;
        }
        __syncthreads();
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            float sk = 0.f, sq = 0.f;
#pragma unroll
            for (int w = 0; w < 8; ++w) {
                sk += part[w * kC + lane + 32 * hf];
                sq += part[8 * kC + w * kC + lane + 32 * hf];
            }
            inv_k[hf] = sk > 0.f ? 1.f / sqrtf(sk) : 0.f;
            inv_q[hf] = sq > 0.f ? 1.f / sqrtf(sq) : 0.f;
            if (warp == 0) {
                sInv[lane + 32 * hf] = inv_k[hf];
                sInv[kC + lane + 32 * hf] = inv_q[hf];
            }
        }
    } else if (warp == 0) {
        sInv[lane] = sInv[lane + 32] = sInv[kC + lane] = sInv[kC + lane + 32] = 1.f;
    }
    __syncthreads();        // the split pass writes over the scratch

    // ---- split operands: Kr, Qr and Kb in shared memory (the Qr and Kb tiles, already in
    // the record's byte order, reach the record by bulk copies once P1 is issued)
    if (!wide_path) {
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
        const int t = lane + 32 * hf;
#pragma unroll
        for (int g = 0; g < 2; ++g) {
            const uint4 kv = kv4[2 * hf + g], qv = qv4[2 * hf + g];
            float kk[8], qq[8], up[8], y[8];
            {
                const __nv_bfloat16 *kb16 = reinterpret_cast<const __nv_bfloat16 *>(&kv);
                const __nv_bfloat16 *qb16 = reinterpret_cast<const __nv_bfloat16 *>(&qv);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    kk[i] = __bfloat162float(kb16[i]) * inv_k[hf];
                    qq[i] = __bfloat162float(qb16[i]) * inv_q[hf];
                }
            }
            const uint32_t ok = core_off(t, ch0 + 8 * g, RW_SO, RW_SI);
            const uint32_t oq = core_off(64 + t, ch0 + 8 * g, RW_SO, RW_SI);
            float gm[8];
            {
                const float4 m0 = reinterpret_cast<const float4 *>(sGm + ch0 + 8 * g)[0];
                const float4 m1 = reinterpret_cast<const float4 *>(sGm + ch0 + 8 * g)[1];
                gm[0] = m0.x; gm[1] = m0.y; gm[2] = m0.z; gm[3] = m0.w;
                gm[4] = m1.x; gm[5] = m1.y; gm[6] = m1.z; gm[7] = m1.w;
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                up[i] = __expf(G[hf][8 * g + i] - gm[i]);
                y[i] = kk[i] * up[i];
            }
            st_split8(smem, PP_P + ok, PP_P_LO + ok, y);                       // Kr
#pragma unroll
            for (int i = 0; i < 8; ++i) y[i] = scale * qq[i] * up[i];
            st_split8(smem, PP_P + oq, PP_P_LO + oq, y);                       // Qr
#pragma unroll
            for (int i = 0; i < 8; ++i) y[i] = kk[i] * __expf(gm[i] - G[hf][8 * g + i]);
            st_split8(smem, PP_KB + ok, PP_KB_LO + ok, y);                     // Kb
        }
    }
    }
    __syncthreads();        // the V region's scalars have been read
    // V (exact bf16; rows past the chunk's end zero-filled) into its operand tile; a
    // wide-range chunk first finishes with the per-token scalars kept in that region
    auto issue_v = [&]() {
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            // eight consecutive threads fill the eight rows of one core matrix (no bank conflicts)
            const int id = tid + kNT * r, t = (id & 7) | ((id >> 7) << 3), g = (id >> 3) & 15;
            const bool okt = t < c;
            cp_async16(sbase + PP_V + core_off(t, 8 * g, RW_SO, RW_SI), v + row(okt ? t : 0) * kDV + 8 * g,
                       okt ? 16u : 0u);
        }
        cp_async_commit();
    };
    if (!wide_path) issue_v();
    if (wide_path) {
        // rare: redo the scan from the inputs and keep G for the pairwise sums; put
        // k e^G, scale q e^G and k e^{G_last - G} where Kr, Qr and Kb were, and set
        // e^m = e^{G_last - m} = 1 in the record
#pragma unroll 1
        for (int hf = 0; hf < 2; ++hf) {
            const int t = lane + 32 * hf;
#pragma unroll 1
            for (int e = 0; e < 16; ++e) {
                const int chn = ch0 + e;
                float a = (t < c) ? la_at(t, chn) : 0.f;
                float a0 = (lane < c) ? la_at(lane, chn) : 0.f;
                if (gate_act) {
                    a = (t < c) ? log_sigmoid(a) : 0.f;
                    a0 = (lane < c) ? log_sigmoid(a0) : 0.f;
                }
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float ua = __shfl_up_sync(0xffffffffu, a, o);
                    const float u0 = __shfl_up_sync(0xffffffffu, a0, o);
                    if (lane >= o) { a += ua; a0 += u0; }
                }
                if (hf) a += __shfl_sync(0xffffffffu, a0, 31);
                reinterpret_cast<float *>(smem + PP_G)[t * kDK + chn] = a;
            }
        }
        if (lane < 16) {
            reinterpret_cast<float *>(rec + R_EM)[ch0 + lane] = 1.f;
            reinterpret_cast<float *>(rec + R_EL)[ch0 + lane] = 1.f;
        }
        __syncthreads();
        const float *sG = reinterpret_cast<const float *>(smem + PP_G);
        for (int id = tid; id < kC * 16; id += kNT) {
            const int t = id >> 4, cg = id & 15;
            float y1[8], y2[8], y3[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int chn = 8 * cg + i;
                const float kk = (t < c) ? __bfloat162float(k[row(t) * kDK + chn]) * sInv[t] : 0.f;
                const float qq = (t < c) ? __bfloat162float(q[row(t) * kDK + chn]) * sInv[kC + t] : 0.f;
                const float gg = sG[t * kDK + chn];
                const float eg = __expf(gg);
                y1[i] = kk * eg;
                y2[i] = scale * qq * eg;
                y3[i] = kk * __expf(sG[(kC - 1) * kDK + chn] - gg);
            }
            const uint32_t ok = core_off(t, 8 * cg, RW_SO, RW_SI);
            const uint32_t oq = core_off(64 + t, 8 * cg, RW_SO, RW_SI);
            st_split8(smem, PP_P + ok, PP_P_LO + ok, y1);
            uint4 hv, lv;
            split8(y2, hv, lv);
            *reinterpret_cast<uint4 *>(rec + R_WQ + oq) = hv;
            *reinterpret_cast<uint4 *>(rec + R_WQ_LO + oq) = lv;
            split8(y3, hv, lv);
            *reinterpret_cast<uint4 *>(rec + R_KT + ok) = hv;
            *reinterpret_cast<uint4 *>(rec + R_KT_LO + ok) = lv;
        }
    }
    proxy_fence();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + PP_TMEMP);
    const uint32_t tlane = (uint32_t)(32 * (warp & 3)) << 16;
    uint32_t phase = 0;
    bool failed = false;

    float *Am = reinterpret_cast<float *>(smem + PP_AMAT);
    if (!wide_path) {
        if (tid == 0) {
            // [Kr; Qr] Kb^T: rows 0..63 -> A, rows 64..127 -> M
            mma_split(tmem + TMP_AM, sbase + PP_P, sbase + PP_P_LO, RW_SI, RW_SO,
                      sbase + PP_KB, sbase + PP_KB_LO, RW_SI, RW_SO, kDK / 16,
                      idesc_bf16(128, 64, 0, 0), false);
            umma_commit(mbar);
            // Qr (rows 64..127 of [Kr; Qr]) and Kb to the record while P1 runs; both
            // tiles are already in the record's byte order, Kb hi and lo contiguous
            bulk_s2g(rec + R_WQ + 16384u, sbase + PP_P + 16384u, 16384u);
            bulk_s2g(rec + R_WQ_LO + 16384u, sbase + PP_P_LO + 16384u, 16384u);
            bulk_s2g(rec + R_KT, sbase + PP_KB, 32768u);
            bulk_commit();
        }
        const bool p1_done = mbar_wait(mbar, phase);
        if (tid == 0) bulk_wait_read();      // the solve's scratch goes over Qr and Kb
        failed = __syncthreads_or(!p1_done) != 0;
        phase ^= 1;
        if (!failed) {
            tc_fence_after();
            float x[32];
            tmem_ld16(tmem + tlane + TMP_AM + 32 * half, *reinterpret_cast<float (*)[16]>(x));
            tmem_ld16(tmem + tlane + TMP_AM + 32 * half + 16, *reinterpret_cast<float (*)[16]>(x + 16));
            if (lrow < 64) {
                const int i = lrow;
                const float bi = sBeta[i];
#pragma unroll
                for (int e4 = 0; e4 < 8; ++e4) {
                    float y[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int j = 32 * half + 4 * e4 + e;
                        y[e] = (j < i) ? bi * x[4 * e4 + e] : 0.f;
                    }
                    *reinterpret_cast<float4 *>(Am + i * kPitch + 32 * half + 4 * e4) = make_float4(y[0], y[1], y[2], y[3]);
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
                    // straight to the record: eight lanes write one core matrix row block,
                    // 128 contiguous bytes
                    const uint32_t o = core_off(i, 32 * half + 8 * g, H_SO, H_SI);
                    uint4 hv, lv;
                    split8(y, hv, lv);
                    *reinterpret_cast<uint4 *>(rec + R_M + o) = hv;
                    *reinterpret_cast<uint4 *>(rec + R_M_LO + o) = lv;
                }
            }
        }
    } else {
        // wide decay range: A and M pair by pair, every factor e^{G_i - G_j} <= 1
        const float *sG = reinterpret_cast<const float *>(smem + PP_G);
        float *Aw = reinterpret_cast<float *>(smem + PP_AW);
        for (int item = tid; item < 2 * 64 * 8; item += kNT) {
            const int isM = item >> 9, i = (item >> 3) & 63, jg = item & 7;
            float y[8];
#pragma unroll 1
            for (int e = 0; e < 8; ++e) {
                const int j = 8 * jg + e;
                float acc = 0.f;
                if (i < c && j < c && (isM ? j <= i : j < i)) {
                    const __nv_bfloat16 *xi = (isM ? q : k) + row(i) * kDK;
                    const __nv_bfloat16 *kj = k + row(j) * kDK;
                    for (int cc = 0; cc < kDK; ++cc)
                        acc += __bfloat162float(xi[cc]) * __bfloat162float(kj[cc]) *
                               __expf(sG[i * kDK + cc] - sG[j * kDK + cc]);
                    acc *= sInv[(isM ? kC : 0) + i] * sInv[j];
                }
                y[e] = isM ? scale * acc : sBeta[i] * acc;
            }
            if (isM) {
                uint4 hv, lv;
                split8(y, hv, lv);
                const uint32_t o = core_off(i, 8 * jg, H_SO, H_SI);
                *reinterpret_cast<uint4 *>(rec + R_M + o) = hv;
                *reinterpret_cast<uint4 *>(rec + R_M_LO + o) = lv;
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) Aw[i * 64 + 8 * jg + e] = y[e];
            }
        }
        __syncthreads();
        issue_v();                           // the per-token scalars are no longer needed
        for (int id = tid; id < 64 * 64; id += kNT) Am[(id >> 6) * kPitch + (id & 63)] = Aw[id];
    }
    __syncthreads();

    if (!failed) {
        // ---- T = (I + A)^-1 by recursive doubling 16 -> 32 -> 64, fp32; R = T Diag(beta)
        float *Tm = reinterpret_cast<float *>(smem + PP_TMAT);
        unit_lower_inverse(Am, Tm, tid);
        __syncthreads();
        for (int id = tid; id < 512; id += kNT) {
            const int i = id >> 3, jg = id & 7;
            const float4 t0v = *reinterpret_cast<const float4 *>(Tm + i * kPitch + 8 * jg);
            const float4 t1v = *reinterpret_cast<const float4 *>(Tm + i * kPitch + 8 * jg + 4);
            const float *bj = sBeta + 8 * jg;
            float y[8] = {t0v.x * bj[0], t0v.y * bj[1], t0v.z * bj[2], t0v.w * bj[3],
                          t1v.x * bj[4], t1v.y * bj[5], t1v.z * bj[6], t1v.w * bj[7]};
            const uint32_t o = core_off(i, 8 * jg, H_SO, H_SI);
            st_split8(smem, PP_R + o, PP_R_LO + o, y);
        }
        cp_async_wait_all();
        proxy_fence();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            // [R; .] Kr (Kr rows read MN-major as B): rows 0..63 are Wr = R Kr;
            // [. ; R] V (R viewed as rows 64..127): rows 64..127 are U, so that the
            // other four warps read it
            mma_split(tmem + TMP_W, sbase + PP_R, sbase + PP_R_LO, H_SI, H_SO,
                      sbase + PP_P, sbase + PP_P_LO, RW_SO, RW_SI, kC / 16,
                      idesc_bf16(128, kDK, 0, 1), false);
            mma_split(tmem + TMP_U, sbase + PP_R - 8192u, sbase + PP_R_LO - 8192u, H_SI, H_SO,
                      sbase + PP_V, 0u, RW_SO, RW_SI, kC / 16,
                      idesc_bf16(128, kDV, 0, 1), false, true, false);
            umma_commit(mbar);
        }
        failed = __syncthreads_or(!mbar_wait(mbar, phase)) != 0;
        phase ^= 1;
        if (!failed) tc_fence_after();
        if (!failed && lrow < 64) {
            // Wr = R Kr: lane = row i, 64 key channels per thread
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                float x[16];
                const int c0 = 64 * half + 16 * r;
                tmem_ld16(tmem + tlane + TMP_W + c0, x);
#pragma unroll
                for (int g = 0; g < 2; ++g) {
                    float y[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) y[e] = x[8 * g + e];
                    // staged in the free [0, 32 KB): hi rows 0..63, then lo
                    const uint32_t o = core_off(lrow, c0 + 8 * g, RW_SO, RW_SI);
                    st_split8(smem, o, 16384u + o, y);
                }
            }
        }
        if (!failed && lrow >= 64) {
            // U: lane 64 + token, 64 value columns per thread = two slices, staged in the
            // free [32 KB, 64 KB) as the swizzled rows of the tensor store's box
#pragma unroll
            for (int s2 = 0; s2 < 2; ++s2) {
                const int r = (2 * half + s2) * kC + lrow - 64;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    float x[16];
                    tmem_ld16(tmem + tlane + TMP_U + 64 * half + 32 * s2 + 16 * hh, x);
#pragma unroll
                    for (int g = 0; g < 4; ++g)
                        *reinterpret_cast<float4 *>(smem + 32768 + u_stage_off(r, 4 * hh + g)) =
                            make_float4(x[4 * g], x[4 * g + 1], x[4 * g + 2], x[4 * g + 3]);
                }
            }
        }
    }

    if (failed && tid == 0) atomicOr(&g_split_device_status, 1u);
    proxy_fence();
    tc_fence_before();
    __syncthreads();
    if (!failed && tid == 0) {
        // Wr (rows 0..63 of [Wr; Qr], hi then lo) and U to the record
        bulk_s2g(rec + R_WQ, sbase, 16384u);
        bulk_s2g(rec + R_WQ_LO, sbase + 16384u, 16384u);
        tma_store_3d(&u_map, sbase + 32768u, 0, 0, bh * nb + nloc);
        bulk_commit();
    }
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem), "r"(TMP_COLS) : "memory");
    }
    if (tid == 0) bulk_wait_read();          // shared memory stays until the copies have read it
}

// ---------------------------------------------------------------- scalar-gate chunk-local kernel
#include "kda_prep_scalar.cuh"

// ---------------------------------------------------------------- chain kernels: modes
// The chain is linear in (U, S_0), which lets one segment of a sequence be run from
// a zero state and corrected afterwards (time-axis split):
constexpr int kChainIdentityS0 = 1;   // start from S = I (dk x dk), ignoring s_in
constexpr int kChainZeroU = 2;        // treat U as zero (propagate the state alone)
constexpr int kChainNoOut = 4;        // write no outputs
constexpr int kChainAccumOut = 8;     // add the outputs to out instead of storing them

// out row slice (16 values) = qs + d3, stored or added
__device__ __forceinline__ void emit_out(float4 *dst, const float (&qs)[16], const float (&d3)[16], bool accum)
{
#pragma unroll
    for (int g = 0; g < 4; ++g) {
        float4 o = make_float4(qs[4 * g] + d3[4 * g], qs[4 * g + 1] + d3[4 * g + 1], qs[4 * g + 2] + d3[4 * g + 2],
                               qs[4 * g + 3] + d3[4 * g + 3]);
        if (accum) {
            const float4 p = dst[g];
            o.x += p.x; o.y += p.y; o.z += p.z; o.w += p.w;
        }
        dst[g] = o;
    }
}

// ---------------------------------------------------------------- chain kernel
// Warp roles: warps 0..7 hold the state slice (thread (lane dk, half) owns 16
// columns of row dk), split the B operands and read the accumulators; warp 8
// issues the tensor-core products; warp 9 issues the record copies (issuing a
// bulk copy stalls the issuing thread for hundreds of cycles, which must not
// delay a product).  Handoffs go through mbarriers, never a CTA-wide barrier:
//   bar_s  (8 arrivals)  S' of chunk kk is in shared memory, D1/D2 of chunk kk-1 read
//   bar_d  (8 arrivals)  Delta of chunk kk is in shared memory, D1 of kk and D3 of kk-1 read
//   mma1 / mma2 (commit) the first product / Kb^T Delta of chunk kk is complete
//   mma3 (commit)        M Delta of chunk kk is complete (the output only: the state
//                        update does not wait for it, it runs beside the next S');
//                        also: Kb and M of chunk kk are no longer read
//   wq_free[s] (commit)  the first product has read the [Wr; Qr] in slot s
// s_in and s_out may be one buffer (the state carried between blocks, or a final
// state written over the initial one): every thread reads its own state elements
// before it writes them, and neither pointer is declared __restrict__.
constexpr int kChainThreads = 320;
constexpr uint32_t CH_WQ = 0;                        // two slots of [Wr; Qr] (hi, lo) and e^m
constexpr uint32_t CH_KTM = 2 * kWqBytes;            // Kb hi, Kb lo, M hi, M lo (48 KB)
constexpr uint32_t CH_MA = CH_KTM + 24576;           // 128-row view whose rows 64..127 are M hi
constexpr uint32_t CH_MA_LO = CH_KTM + 32768;        //   ... and M lo
constexpr uint32_t CH_GAM = CH_KTM + 49152;          // fp32 [128] e^{G_last}, then [128] e^{G_last - m}
constexpr uint32_t CH_S = CH_GAM + 1024, CH_S_LO = CH_S + 8192;    // S': MN-major B (outer dk, inner column)
constexpr uint32_t CH_DL = CH_S + 16384, CH_DL_LO = CH_DL + 4096;  // Delta: MN-major B (outer token)
constexpr uint32_t CH_MBAR = CH_DL + 8192;           // mma1, mma2, wq[2], ktm, bar_s, bar_d
constexpr uint32_t CH_FAIL = CH_MBAR + 56;           // a wait gave up somewhere in the CTA
constexpr uint32_t CH_TMEMP = CH_MBAR + 64;
constexpr uint32_t CH_MBAR3 = CH_MBAR + 72;          // mma3
constexpr uint32_t CH_WQFREE = CH_MBAR + 80;         // wq_free[2]
constexpr uint32_t CH_TOTAL = CH_MBAR + 96;
static_assert(CH_TOTAL <= 232448, "shared memory");
static_assert(R_KT_LO + 16384 == R_M && R_M + 16384 == R_U, "Kb and M are one contiguous copy");
static_assert(R_GAM + 512 == R_EL, "e^{G_last} and e^{G_last - m} are one contiguous copy");

constexpr uint32_t TMC_D1 = 0, TMC_D2 = 32, TMC_D3 = 64, TMC_COLS = 128;

__global__ void __launch_bounds__(kChainThreads, 1)
prefill_chain_kernel(const uint8_t *__restrict__ ws, const float *s_in,
                     float *s_out, float *__restrict__ out, int T, int H, int n0, int nb,
                     int mode, const float *__restrict__ s_add)
{
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t sbase = (uint32_t)__cvta_generic_to_shared(smem);
    const float *sGam = reinterpret_cast<const float *>(smem + CH_GAM);
    volatile uint32_t *sFail = reinterpret_cast<volatile uint32_t *>(smem + CH_FAIL);
    const uint32_t mbar1 = sbase + CH_MBAR, mbar2 = mbar1 + 8, mbar_wq0 = mbar1 + 16, mbar_ktm = mbar1 + 32;
    const uint32_t bar_s = mbar1 + 40, bar_d = mbar1 + 48, mbar3 = sbase + CH_MBAR3;
    const uint32_t wq_free0 = sbase + CH_WQFREE;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int slice = blockIdx.x % kNSL;
    const int bh = blockIdx.x / kNSL;
    const int b = bh / H, h = bh % H;
    const int col0 = slice * kDVS;
    const int lrow = 32 * (warp & 3) + lane;
    const int half = (warp >> 2) & 1;
    const uint8_t *recs = ws + (size_t)bh * nb * kRec;

    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     :: "r"(sbase + CH_TMEMP), "r"(TMC_COLS) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (tid == 0) {
        mbar_init(mbar1, 1);
        mbar_init(mbar2, 1);
        mbar_init(mbar3, 1);
        mbar_init(mbar_wq0, 1);
        mbar_init(mbar_wq0 + 8, 1);
        mbar_init(wq_free0, 1);
        mbar_init(wq_free0 + 8, 1);
        mbar_init(mbar_ktm, 1);
        mbar_init(bar_s, 8);
        mbar_init(bar_d, 8);
        *sFail = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + CH_TMEMP);
    // a wait that gives up marks the CTA failed; the others then stop at their next wait
    auto wait = [&](uint32_t bar, uint32_t parity) -> bool {
        if (mbar_try(bar, parity)) return true;        // fast path: no flag read, no clock
        if (*sFail) return false;
        if (mbar_wait(bar, parity)) return true;
        *sFail = 1u;
        return false;
    };

    if (warp == 8) {
        // ---------------- issuer: the products (lane 0)
        if (lane == 0) {
            for (int kk = 0; kk < nb; ++kk) {
                const uint32_t par = (uint32_t)kk & 1u;
                // S' written; the compute warps have waited for this chunk's [Wr; Qr]
                if (!wait(bar_s, par)) break;
                tc_fence_after();
                const uint32_t wq = sbase + CH_WQ + kWqBytes * (kk & 1);
                mma_split(tmem + TMC_D1, wq, wq + 32768u, RW_SI, RW_SO, sbase + CH_S, sbase + CH_S_LO,
                          S_SO, S_SI, kDK / 16, idesc_bf16(128, kDVS, 0, 1), false);
                umma_commit(mbar1);
                umma_commit(wq_free0 + 8u * (kk & 1));
                // Delta written; the compute warps have waited for this chunk's Kb, M, decays
                if (!wait(bar_d, par)) break;
                tc_fence_after();
                mma_split(tmem + TMC_D2, sbase + CH_KTM, sbase + CH_KTM + 16384u, RW_SO, RW_SI,
                          sbase + CH_DL, sbase + CH_DL_LO, S_SO, S_SI, kC / 16, idesc_bf16(128, kDVS, 1, 1), false);
                umma_commit(mbar2);
                mma_split(tmem + TMC_D3, sbase + CH_MA, sbase + CH_MA_LO, H_SI, H_SO,
                          sbase + CH_DL, sbase + CH_DL_LO, S_SO, S_SI, kC / 16, idesc_bf16(128, kDVS, 0, 1), false);
                umma_commit(mbar3);
            }
        }
    } else if (warp == 9) {
        // ---------------- copies (lane 0): [Wr; Qr] and e^m two chunks ahead (two slots,
        // refilled once the first product has read them), Kb, M and the decays one chunk
        // ahead (one slot, refilled once both products of the chunk have read it).
        // Every refill waits for the slot's previous use, so no wait here can fall two
        // phases behind its barrier.
        if (lane == 0) {
            uint32_t wq_pend = 0u, wq_par = 0u, ktm_par = 0u;
            bool ktm_pending = false;
            auto load_wq = [&](int kk) {
                const uint32_t mb = mbar_wq0 + 8u * (kk & 1);
                const uint32_t bit = 1u << (kk & 1);
                wq_pend |= bit;
                wq_par = ((kk >> 1) & 1) ? (wq_par | bit) : (wq_par & ~bit);
                mbar_expect_tx(mb, kWqBytes);
                bulk_g2s(sbase + CH_WQ + kWqBytes * (kk & 1), recs + (size_t)kk * kRec + R_WQ, kWqBytes, mb);
            };
            auto load_ktm = [&](int kk) {
                const uint8_t *r = recs + (size_t)kk * kRec;
                ktm_pending = true;
                ktm_par = (uint32_t)kk & 1u;
                mbar_expect_tx(mbar_ktm, 49152u + 1024u);
                bulk_g2s(sbase + CH_KTM, r + R_KT, 49152u, mbar_ktm);
                bulk_g2s(sbase + CH_GAM, r + R_GAM, 1024u, mbar_ktm);
            };
            load_wq(0);
            if (nb > 1) load_wq(1);
            load_ktm(0);
            for (int kk = 0; kk < nb; ++kk) {
                if (kk + 2 < nb) {
                    if (!wait(wq_free0 + 8u * (kk & 1), (uint32_t)(kk >> 1) & 1u)) break;
                    wq_pend &= ~(1u << (kk & 1));
                    load_wq(kk + 2);
                }
                if (kk + 1 < nb) {
                    if (!wait(mbar3, (uint32_t)kk & 1u)) break;
                    load_ktm(kk + 1);
                }
            }
            if (*sFail) {
                // let the copies still in flight land before shared memory is released
                for (int sl = 0; sl < 2; ++sl)
                    if ((wq_pend >> sl) & 1u) mbar_wait(mbar_wq0 + 8u * sl, (wq_par >> sl) & 1u);
                if (ktm_pending) mbar_wait(mbar_ktm, ktm_par);
            }
        }
    } else {
        // ---------------- state slice: S' and Delta operands, updates, outputs
        const uint32_t tlane = (uint32_t)(32 * (warp & 3)) << 16;
        float S[16];
#pragma unroll
        for (int j = 0; j < 16; ++j)
            S[j] = (mode & kChainIdentityS0) ? (lrow == col0 + 16 * half + j ? 1.f : 0.f)
                   : s_in ? s_in[((size_t)bh * kDK + lrow) * kDV + col0 + 16 * half + j] : 0.f;
        float qs[16];
        bool ok = true;
        for (int kk = 0; kk < nb && ok; ++kk) {
            const uint32_t par = (uint32_t)kk & 1u;
            // this thread's 16 values of U (token lrow), read from the record into
            // registers now and used after the first product
            float uu[16];
            if (lrow < 64 && !(mode & kChainZeroU)) {
                const float4 *src = reinterpret_cast<const float4 *>(recs + (size_t)kk * kRec + R_U + slice * 8192u +
                                                                     lrow * 128u + half * 64u);
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    const float4 u4 = src[g];
                    uu[4 * g] = u4.x; uu[4 * g + 1] = u4.y; uu[4 * g + 2] = u4.z; uu[4 * g + 3] = u4.w;
                }
            } else {
#pragma unroll
                for (int e = 0; e < 16; ++e) uu[e] = 0.f;
            }
            // ---- S' = Diag(e^m) S of chunk kk as a split B operand
            if (!(ok = wait(mbar_wq0 + 8u * (kk & 1), (uint32_t)(kk >> 1) & 1u))) break;
            {
                const float em = reinterpret_cast<const float *>(smem + CH_WQ + kWqBytes * (kk & 1) + 65536u)[lrow];
#pragma unroll
                for (int g = 0; g < 2; ++g) {
                    float xv[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) xv[e] = em * S[8 * g + e];
                    const uint32_t off = core_off(lrow, 16 * half + 8 * g, S_SO, S_SI);
                    st_split8(smem, CH_S + off, CH_S_LO + off, xv);
                }
            }
            proxy_fence();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_s);

            // ---- O = Qr S' + M Delta of chunk kk - 1 while the first product of kk runs
            if (kk > 0 && lrow >= 64) {
                if (!(ok = wait(mbar3, par ^ 1u))) break;
                tc_fence_after();
                float o2[16];
                tmem_ld16(tmem + tlane + TMC_D3 + 16 * half, o2);
                const int t = (n0 + kk - 1) * kC + lrow - 64;
                if (t < T && !(mode & kChainNoOut))
                    emit_out(reinterpret_cast<float4 *>(out + (((size_t)b * T + t) * H + h) * kDV + col0 + 16 * half),
                             qs, o2, (mode & kChainAccumOut) != 0);
            }

            // ---- Delta = U - Wr S' (rows 0..63); Qr S' kept for the output (rows 64..127)
            if (!(ok = wait(mbar1, par) && wait(mbar_ktm, par))) break;
            tc_fence_after();
            {
                float x[16];
                tmem_ld16(tmem + tlane + TMC_D1 + 16 * half, x);
                if (lrow < 64) {
#pragma unroll
                    for (int g = 0; g < 2; ++g) {
                        float d[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            d[e] = uu[8 * g + e] - x[8 * g + e];
                        const uint32_t o = core_off(lrow, 16 * half + 8 * g, S_SO, S_SI);
                        st_split8(smem, CH_DL + o, CH_DL_LO + o, d);
                    }
                }
#pragma unroll
                for (int e = 0; e < 16; ++e) qs[e] = x[e];
            }
            const float gam = sGam[lrow], el = sGam[kDK + lrow];
            proxy_fence();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_d);

            // ---- S <- Diag(e^{G_last}) S + Diag(e^{G_last - m}) Kb^T Delta
            if (!(ok = wait(mbar2, par))) break;
            tc_fence_after();
            {
                float x[16];
                tmem_ld16(tmem + tlane + TMC_D2 + 16 * half, x);
#pragma unroll
                for (int j = 0; j < 16; ++j) S[j] = gam * S[j] + el * x[j];
            }
            tc_fence_before();
        }
        if (ok && nb > 0 && lrow >= 64 && (ok = wait(mbar3, (uint32_t)(nb - 1) & 1u))) {
            // the last chunk's output
            tc_fence_after();
            float o2[16];
            tmem_ld16(tmem + tlane + TMC_D3 + 16 * half, o2);
            const int t = (n0 + nb - 1) * kC + lrow - 64;
            if (t < T && !(mode & kChainNoOut))
                emit_out(reinterpret_cast<float4 *>(out + (((size_t)b * T + t) * H + h) * kDV + col0 + 16 * half),
                         qs, o2, (mode & kChainAccumOut) != 0);
        }
        if (ok && s_out) {
            const size_t o = ((size_t)bh * kDK + lrow) * kDV + col0 + 16 * half;
            if (s_add) {
#pragma unroll
                for (int j = 0; j < 16; ++j) S[j] += s_add[o + j];
            }
            float4 *dst = reinterpret_cast<float4 *>(s_out + o);
#pragma unroll
            for (int g = 0; g < 4; ++g) dst[g] = make_float4(S[4 * g], S[4 * g + 1], S[4 * g + 2], S[4 * g + 3]);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (tid == 0 && *sFail) atomicOr(&g_split_device_status, 1u);
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem), "r"(TMC_COLS) : "memory");
    }
}

// ---------------------------------------------------------------- per-head chain kernel
// The chain of one (b, h) with all 128 value columns in one CTA, the state held
// transposed: thread (warp w < 16, lane l) owns value column c = 32 (w % 4) + l (its
// tensor-memory lane) and key channels 32 (w / 4) .. + 31 of S^T, in registers.  With
// the value axis on the tensor-memory lanes, S'^T and Delta^T are A operands read from
// tensor memory, and the records' tiles serve unchanged as B operands:
//   D1^T = S'^T [Wr; Qr]^T        (M = 128 values, N = 128 rows, K = dk)
//   Delta^T = U^T - D1^T[:, 0:64]
//   D2^T = Delta^T Kb             (N = dk, K = tokens)
//   D3^T = Delta^T M^T            (N = 64 output tokens)
//   O^T = D1^T[:, 64:128] + D3^T,   S^T <- S^T Diag(e^{G_last}) + D2^T Diag(e^{G_last - m})
// Every product is N = 64 or 128 wide, so one CTA per head walks a chunk in about the
// time a 32-column slice CTA does, on a quarter of the SMs; and shared memory holds
// only records: [Wr; Qr] in two slots (two chunks ahead), Kb, M, U and the decays in one.
// A chunk's outputs are staged in the hi half of its [Wr; Qr] slot once D1 has read it
// and leave by one TMA tensor store (plain stores from 512 threads slowed the next
// chunk's D1 by a third); the slot's lo half and e^m are refilled as soon as D1 is
// done, the hi half once the store has read it.  Warp 16 issues the products; warp 17 the record copies, the output stores
// and L2 prefetches.  Handoffs are mbarriers (one arrival per compute warp):
//   bar_s  S'^T of chunk kk is in tensor memory (and D1 of kk - 1 has been read back):
//          two barriers, the K steps of key channels 32 j + 0..15 (even) first, then
//          32 j + 16..31 (odd), so that D1 starts on the first half while the second
//          is still being split
//   bar_d  Delta^T of chunk kk is in tensor memory (and D3 of kk - 1 has been read back)
//   bar_u  the state update of chunk kk has read its decays from the Kb/M slot
//   out_st the outputs of chunk kk are staged in its [Wr; Qr] slot (so D1 and D3 of kk
//          are complete)
//   mma1 / mma2 / mma3 (commit)  D1 / D2 / D3 of chunk kk complete
constexpr int kTThreads = 18 * 32;
constexpr uint32_t TC_WQ = 0;                         // two slots of [Wr; Qr] hi, lo, e^m
constexpr uint32_t TC_KTM = 2 * kWqBytes;             // Kb hi, Kb lo, M hi, M lo, then the decays
constexpr uint32_t TC_DEC = TC_KTM + 49152;           // e^{G_last} [128], e^{G_last - m} [128]
constexpr uint32_t TC_U = TC_DEC + 1024;              // U fp32 [value slice][token][32]
constexpr uint32_t TC_MBAR = TC_U + 32768;            // mma1, mma2, mma3, wq_lo[2], wq_hi[2], ktm, bar_s, bar_d, bar_u
constexpr uint32_t TC_FAIL = TC_MBAR + 88;
constexpr uint32_t TC_TMEMP = TC_MBAR + 96;
constexpr uint32_t TC_OUTST = TC_MBAR + 104;          // out_st
constexpr uint32_t TC_BARS1 = TC_MBAR + 112;          // bar_s1 (S'^T odd K steps)
constexpr uint32_t TC_TOTAL = TC_MBAR + 120;
static_assert(TC_TOTAL <= 232448, "shared memory");
// tensor-memory columns (lane = value column)
constexpr uint32_t TT_S = 0, TT_S_LO = 64;            // S'^T, bf16 pairs along dk: hi, lo
constexpr uint32_t TT_DL = 128, TT_DL_LO = 160;       // Delta^T, bf16 pairs along tokens: hi, lo
constexpr uint32_t TT_D3 = 192, TT_D1 = 256, TT_D2 = 384, TT_COLS = 512;

// kScalar: records of the scalar-gate chunk-local kernel (e^m = e^{G_last - m} = 1 and
// one e^{G_last} in every channel), so the state update is one multiply-add per value
// and S'^T = S^T.
template <bool kScalar>
__global__ void __launch_bounds__(kTThreads, 1)
prefill_chain_t_kernel(const uint8_t *__restrict__ ws, const float *s_in, float *s_out,
                       const __grid_constant__ CUtensorMap out_map, int T, int H, int n0, int nb, int mode,
                       const float *__restrict__ s_add)
{
    // a chunk-local launch made programmatically dependent on this one may place its CTAs
    // once every CTA of this grid is resident: they go to the SMs this grid leaves free
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t sbase = (uint32_t)__cvta_generic_to_shared(smem);
    volatile uint32_t *sFail = reinterpret_cast<volatile uint32_t *>(smem + TC_FAIL);
    // [Wr; Qr] slots arrive in two halves: lo with e^m (wq_lo), then hi (wq_hi), whose
    // region also stages the outputs
    const uint32_t mbar1 = sbase + TC_MBAR, mbar2 = mbar1 + 8, mbar3 = mbar1 + 16, wq_lo0 = mbar1 + 24;
    const uint32_t wq_hi0 = mbar1 + 40, mbar_ktm = mbar1 + 56, bar_s = mbar1 + 64, bar_d = mbar1 + 72;
    const uint32_t bar_u = mbar1 + 80, out_st = sbase + TC_OUTST, bar_s1 = sbase + TC_BARS1;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.x;
    const int b = bh / H, h = bh % H;
    const uint8_t *recs = ws + (size_t)bh * nb * kRec;

    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     :: "r"(sbase + TC_TMEMP), "r"(TT_COLS) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (tid == 0) {
        mbar_init(mbar1, 1);
        mbar_init(mbar2, 1);
        mbar_init(mbar3, 1);
        mbar_init(wq_lo0, 1);
        mbar_init(wq_lo0 + 8, 1);
        mbar_init(wq_hi0, 1);
        mbar_init(wq_hi0 + 8, 1);
        mbar_init(mbar_ktm, 1);
        mbar_init(bar_s, 16);
        mbar_init(bar_s1, 16);
        mbar_init(bar_d, 16);
        mbar_init(bar_u, 16);
        mbar_init(out_st, 16);
        *sFail = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + TC_TMEMP);
    // a wait that gives up marks the CTA failed; the others then stop at their next wait
    auto wait = [&](uint32_t bar, uint32_t parity) -> bool {
        if (mbar_try(bar, parity)) return true;        // fast path: no flag read, no clock
        if (*sFail) return false;
        if (mbar_wait(bar, parity)) return true;
        *sFail = 1u;
        return false;
    };

    if (warp == 16) {
        // ---------------- issuer: the products (lane 0)
        if (lane == 0) {
            const uint32_t id1 = idesc_bf16(128, 2 * kC, 0, 0);    // B = [Wr; Qr], K-major (rows, dk)
            const uint32_t id2 = idesc_bf16(128, kDK, 0, 1);       // B = Kb, MN-major (token, dk)
            const uint32_t id3 = idesc_bf16(128, kC, 0, 0);        // B = M^T, K-major (output token, token)
            for (int kk = 0; kk < nb; ++kk) {
                const uint32_t par = (uint32_t)kk & 1u;
                if (!wait(bar_s, par) || !wait(wq_hi0 + 8u * (kk & 1), (uint32_t)(kk >> 1) & 1u)) break;
                tc_fence_after();
                const uint32_t wq = sbase + TC_WQ + kWqBytes * (kk & 1);
                // the even K steps (key channels 32 j .. + 15) while the odd ones are split
                mma_split_ta_steps(tmem + TT_D1, tmem + TT_S, tmem + TT_S_LO, wq, wq + 32768u, RW_SI, RW_SO, 0, 2,
                                   kDK / 32, id1, false);
                if (!wait(bar_s1, par)) break;
                tc_fence_after();
                mma_split_ta_steps(tmem + TT_D1, tmem + TT_S, tmem + TT_S_LO, wq, wq + 32768u, RW_SI, RW_SO, 1, 2,
                                   kDK / 32, id1, true);
                umma_commit(mbar1);
                if (!wait(bar_d, par)) break;
                tc_fence_after();
                mma_split_ta(tmem + TT_D2, tmem + TT_DL, tmem + TT_DL_LO, sbase + TC_KTM, sbase + TC_KTM + 16384u,
                             RW_SO, RW_SI, kC / 16, id2);
                umma_commit(mbar2);
                mma_split_ta(tmem + TT_D3, tmem + TT_DL, tmem + TT_DL_LO, sbase + TC_KTM + 32768u,
                             sbase + TC_KTM + 40960u, H_SI, H_SO, kC / 16, id3);
                umma_commit(mbar3);
            }
        }
    } else if (warp == 17) {
        // ---------------- copies (lane 0): [Wr; Qr] and e^m two chunks ahead (two slots,
        // refilled once the outputs staged there have left); Kb, M, U and the decays one
        // chunk ahead (one slot, refilled once D2 and D3 have read it and the state update
        // has read the decays); the outputs of each chunk by one tensor store (or
        // reduce-add); the whole record three chunks ahead prefetched into L2
        if (lane == 0) {
            uint32_t pend = 0u, par_bits = 0u, ktm_par = 0u;   // bit 2 s + h: slot s, half h (1 = hi) in flight
            bool ktm_pending = false;
            auto load_half = [&](int kk, int hi) {
                const int sl = kk & 1;
                const uint32_t mb = (hi ? wq_hi0 : wq_lo0) + 8u * sl;
                const uint32_t bit = 1u << (2 * sl + hi);
                pend |= bit;
                par_bits = ((kk >> 1) & 1) ? (par_bits | bit) : (par_bits & ~bit);
                const uint32_t off = hi ? 0u : 32768u, bytes = hi ? 32768u : kWqBytes - 32768u;
                mbar_expect_tx(mb, bytes);
                bulk_g2s(sbase + TC_WQ + kWqBytes * sl + off, recs + (size_t)kk * kRec + R_WQ + off, bytes, mb);
            };
            auto load_ktm = [&](int kk) {
                const uint8_t *r = recs + (size_t)kk * kRec;
                ktm_pending = true;
                ktm_par = (uint32_t)kk & 1u;
                mbar_expect_tx(mbar_ktm, 49152u + 1024u + 32768u);
                bulk_g2s(sbase + TC_KTM, r + R_KT, 49152u, mbar_ktm);
                bulk_g2s(sbase + TC_DEC, r + R_GAM, 1024u, mbar_ktm);
                bulk_g2s(sbase + TC_U, r + R_U, 32768u, mbar_ktm);
            };
            auto prefetch = [&](int kk) {
                const uint8_t *r = recs + (size_t)kk * kRec;
                for (uint32_t o = 0; o < kRec; o += 32768u)
                    l2_prefetch(r + o, (kRec - o) < 32768u ? (kRec - o) : 32768u);
            };
            // chunk 0's slot and Kb/M/U first (its S'^T split, D1 and Delta wait for
            // them), then the L2 prefetches and chunk 1's slot
            load_half(0, 0);
            load_half(0, 1);
            load_ktm(0);
            for (int kk = 1; kk < 3 && kk < nb; ++kk) prefetch(kk);
            if (nb > 1) {
                load_half(1, 0);
                load_half(1, 1);
            }
            for (int kk = 0; kk < nb; ++kk) {
                if (kk + 3 < nb) prefetch(kk + 3);
                // D3 done (so D2 and D1 too) and the decays read: the Kb/M slot refills first
                // (the next Delta waits for it), then slot kk % 2's lo half and e^m
                if (!wait(mbar3, (uint32_t)kk & 1u)) break;
                pend &= ~(1u << (2 * (kk & 1)));
                if (kk + 1 < nb) {
                    if (!wait(bar_u, (uint32_t)kk & 1u)) break;
                    load_ktm(kk + 1);
                }
                if (kk + 2 < nb) load_half(kk + 2, 0);
                // the outputs of kk, staged in the slot's hi half, leave by one tensor store
                if (!wait(out_st, (uint32_t)kk & 1u)) break;
                pend &= ~(1u << (2 * (kk & 1) + 1));
                if (!(mode & kChainNoOut)) {
                    const uint32_t src = sbase + TC_WQ + kWqBytes * (kk & 1);
                    if (mode & kChainAccumOut) tma_reduce_add_4d(&out_map, src, 0, h, (n0 + kk) * kC, b);
                    else tma_store_4d(&out_map, src, 0, h, (n0 + kk) * kC, b);
                    bulk_commit();
                }
                if (kk + 2 < nb) {
                    bulk_wait_read();                  // the outputs have left the hi half
                    load_half(kk + 2, 1);
                }
            }
            bulk_wait_read();
            if (*sFail) {
                // let the copies still in flight land before shared memory is released
                for (int sl = 0; sl < 2; ++sl)
                    for (int hi = 0; hi < 2; ++hi)
                        if ((pend >> (2 * sl + hi)) & 1u)
                            mbar_wait((hi ? wq_hi0 : wq_lo0) + 8u * sl, (par_bits >> (2 * sl + hi)) & 1u);
                if (ktm_pending) mbar_wait(mbar_ktm, ktm_par);
            }
        }
    } else {
        // ---------------- state: value column c, key channels i0 .. i0 + 31
        const int q4 = warp & 3, g = warp >> 2;
        const int c = 32 * q4 + lane;
        const int i0 = 32 * g;
        const uint32_t tlane = (uint32_t)(32 * q4) << 16;
        const float *sDec = reinterpret_cast<const float *>(smem + TC_DEC);
        float S[32];
#pragma unroll
        for (int j = 0; j < 32; ++j)
            S[j] = (mode & kChainIdentityS0) ? (i0 + j == c ? 1.f : 0.f)
                   : s_in ? s_in[((size_t)bh * kDK + i0 + j) * kDV + c] : 0.f;
        // S'^T = S^T Diag(e^m) of chunk kk as the hi/lo A operand (pairs of key channels)
        auto put_s = [&](int kk) -> bool {
            if (!wait(wq_lo0 + 8u * (kk & 1), (uint32_t)(kk >> 1) & 1u)) return false;
            const float4 *em4 = reinterpret_cast<const float4 *>(smem + TC_WQ + kWqBytes * (kk & 1) + 65536u) + i0 / 4;
            uint32_t hv[16], lv[16];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float2 s01 = make_float2(S[4 * e], S[4 * e + 1]), s23 = make_float2(S[4 * e + 2], S[4 * e + 3]);
                if (kScalar) {
                    split_pair2(s01, hv[2 * e], lv[2 * e]);
                    split_pair2(s23, hv[2 * e + 1], lv[2 * e + 1]);
                } else {
                    const float4 m = em4[e];
                    split_pair2(mul2(make_float2(m.x, m.y), s01), hv[2 * e], lv[2 * e]);
                    split_pair2(mul2(make_float2(m.z, m.w), s23), hv[2 * e + 1], lv[2 * e + 1]);
                }
            }
            tmem_st16u(tmem + tlane + TT_S + 16 * g, hv);
            tmem_st16u(tmem + tlane + TT_S_LO + 16 * g, lv);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(bar_s);
                mbar_arrive(bar_s1);
            }
            return true;
        };
        // this thread's 16 outputs of chunk kk (value column c, tokens 16 g .. + 15): Qr S'
        // from D1, then D3 added and the sum staged for the tensor store
        float o[16];
        bool ok = true;
        if (nb > 0) ok = put_s(0);
        for (int kk = 0; kk < nb && ok; ++kk) {
            const uint32_t par = (uint32_t)kk & 1u;

            // ---- Delta^T = U^T - D1^T[:, 0:64] for tokens 16 g .. 16 g + 15; Qr S' kept
            if (!(ok = wait(mbar1, par) && wait(mbar_ktm, par))) break;
            tc_fence_after();
            {
                float x[16];
                tmem_ld16(tmem + tlane + TT_D1 + 16 * g, x);
                // U: value column c of tokens 16 g .. 16 g + 15 ([slice][token][32] in the slot)
                const float *su = reinterpret_cast<const float *>(smem + TC_U) + q4 * 2048 + (16 * g) * kDVS + lane;
                const bool zu = (mode & kChainZeroU) != 0;
                uint32_t hv[8], lv[8];
#pragma unroll
                for (int p = 0; p < 8; ++p) {
                    const float u0 = zu ? 0.f : su[(2 * p) * kDVS], u1 = zu ? 0.f : su[(2 * p + 1) * kDVS];
                    split_pair2(sub2(make_float2(u0, u1), make_float2(x[2 * p], x[2 * p + 1])), hv[p], lv[p]);
                }
                tmem_st8u(tmem + tlane + TT_DL + 8 * g, hv);
                tmem_st8u(tmem + tlane + TT_DL_LO + 8 * g, lv);
                tmem_wait_st();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_d);
            // Qr S' of this thread's outputs, read while D2 runs (D1's columns stay until the
            // next chunk's D1, which waits for this chunk's S'^T handoff)
            tmem_ld16(tmem + tlane + TT_D1 + 64 + 16 * g, o);

            // ---- S^T <- S^T Diag(e^{G_last}) + D2^T Diag(e^{G_last - m}), and in the same pass
            // the next chunk's S'^T = S^T Diag(e^m') (its e^m arrived two chunks ahead)
            if (!(ok = wait(mbar2, par))) break;
            const bool next = kk + 1 < nb;
            if (next && !(ok = wait(wq_lo0 + 8u * ((kk + 1) & 1), (uint32_t)((kk + 1) >> 1) & 1u))) break;
            tc_fence_after();
            {
                const float4 *em4 =
                    reinterpret_cast<const float4 *>(smem + TC_WQ + kWqBytes * ((kk + 1) & 1) + 65536u) + i0 / 4;
                const float gam_s = sDec[0];
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    float x[16];
                    tmem_ld16(tmem + tlane + TT_D2 + i0 + 16 * hh, x);
                    const float4 *gam4 = reinterpret_cast<const float4 *>(sDec + i0 + 16 * hh);
                    const float4 *el4 = reinterpret_cast<const float4 *>(sDec + kDK + i0 + 16 * hh);
                    uint32_t hv[8], lv[8];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        float *sv = S + 16 * hh + 4 * e;
                        const float2 x01 = make_float2(x[4 * e], x[4 * e + 1]), x23 = make_float2(x[4 * e + 2], x[4 * e + 3]);
                        float2 s01 = make_float2(sv[0], sv[1]), s23 = make_float2(sv[2], sv[3]);
                        if (kScalar) {
                            const float2 gg = make_float2(gam_s, gam_s);
                            s01 = fma2(gg, s01, x01);
                            s23 = fma2(gg, s23, x23);
                            if (next) {
                                split_pair2(s01, hv[2 * e], lv[2 * e]);
                                split_pair2(s23, hv[2 * e + 1], lv[2 * e + 1]);
                            }
                        } else {
                            const float4 ga = gam4[e], el = el4[e];
                            s01 = fma2(make_float2(ga.x, ga.y), s01, mul2(make_float2(el.x, el.y), x01));
                            s23 = fma2(make_float2(ga.z, ga.w), s23, mul2(make_float2(el.z, el.w), x23));
                            if (next) {
                                const float4 m = em4[4 * hh + e];
                                split_pair2(mul2(make_float2(m.x, m.y), s01), hv[2 * e], lv[2 * e]);
                                split_pair2(mul2(make_float2(m.z, m.w), s23), hv[2 * e + 1], lv[2 * e + 1]);
                            }
                        }
                        sv[0] = s01.x; sv[1] = s01.y; sv[2] = s23.x; sv[3] = s23.y;
                    }
                    if (next) {
                        tmem_st8u(tmem + tlane + TT_S + 16 * g + 8 * hh, hv);
                        tmem_st8u(tmem + tlane + TT_S_LO + 16 * g + 8 * hh, lv);
                        tmem_wait_st();
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(hh == 0 ? bar_s : bar_s1);
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_u);      // the decays are read: the Kb/M slot may refill
            }

            // ---- O = Qr S' + M Delta of this chunk, staged row-major [token][value] in its
            // [Wr; Qr] slot (read by D1, which is complete), for the copy warp's tensor store;
            // after the next chunk's handoff, off the critical path
            if (!(ok = wait(mbar3, par))) break;
            tc_fence_after();
            {
                float x[16];
                tmem_ld16(tmem + tlane + TT_D3 + 16 * g, x);
                float *so = reinterpret_cast<float *>(smem + TC_WQ + kWqBytes * (kk & 1)) + (16 * g) * kDV + c;
#pragma unroll
                for (int j = 0; j < 16; ++j) so[j * kDV] = o[j] + x[j];
            }
            proxy_fence();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(out_st);
        }
        if (ok && s_out) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const size_t o = ((size_t)bh * kDK + i0 + j) * kDV + c;
                s_out[o] = s_add ? S[j] + s_add[o] : S[j];
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (tid == 0 && *sFail) atomicOr(&g_split_device_status, 1u);
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem), "r"(TT_COLS) : "memory");
    }
}

// ---------------------------------------------------------------- failure-path self-test
// One CTA waits on an mbarrier phase that nothing completes, with the bounded wait
// of the kernels above but a caller-chosen limit; giving up records the same status
// bit the prefill kernels record.
__global__ void selftest_timeout_kernel(long long limit_cycles)
{
    __shared__ __align__(8) uint64_t bar;
    const uint32_t addr = (uint32_t)__cvta_generic_to_shared(&bar);
    if (threadIdx.x == 0) {
        mbar_init(addr, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    const bool ok = mbar_wait(addr, 0u, limit_cycles);
    if (!ok && threadIdx.x == 0) atomicOr(&g_split_device_status, 1u);
}

}  // namespace

bool prefill_split_supported(const ForwardArgs &a)
{
    // any gate: a scalar decay (or none) is staged as the same value in every channel
    return a.dtype == KDA_BF16 && a.dk == kDK && a.dv == kDV &&
           (a.gate == KDA_GATE_CHANNEL || a.prep_flags == 0);
}

size_t prefill_split_workspace_full(int B, int T, int H)
{
    const size_t nchunks = ((size_t)T + kC - 1) / kC;
    return (size_t)B * H * nchunks * kRec;
}

namespace {

// The pipelined schedule: blocks of up to kPipeChunks chunks whose records alternate
// between two workspace slots, so that the chunk-local kernel fills the next block
// while the per-head chain walks the current one on its own SMs.
constexpr int kPipeChunks = 64, kPipeMinChunks = 8;

int device_sms()
{
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
                                                  cudaSuccess || sms <= 0) {
        cudaGetLastError();         // no device here: size the schedule for a B200
        return 148;
    }
    return sms;
}

// A shape that takes the pipelined schedule: the per-head chain leaves at least half
// the SMs to the chunk-local kernel, and the sequence has two full blocks.
bool pipelined_shape(size_t bh, size_t nch, int sms)
{
    return 2 * bh <= (size_t)sms && nch >= 2 * (size_t)kPipeChunks;
}

}  // namespace

// Which chain kernel a problem runs, from the shape of its whole sequence, so that
// every schedule of one problem (any workspace, the host-memory path) does the same
// arithmetic: one CTA per (b, h) when the heads alone fill the SMs or the schedule is
// pipelined, else one CTA per (b, h, 32-column slice).
bool split_per_head(int B, int T_whole, int H)
{
    const size_t bh = (size_t)B * H, nch = ((size_t)T_whole + kC - 1) / kC;
    const int sms = device_sms();
    return bh * kNSL > (size_t)sms || pipelined_shape(bh, nch, sms);
}

size_t prefill_split_workspace_best(int B, int T, int H)
{
    const size_t bh = (size_t)B * H, nch = ((size_t)T + kC - 1) / kC;
    if (pipelined_shape(bh, nch, device_sms()))
        return 2 * (size_t)kPipeChunks * bh * kRec + bh * kDK * kDV * sizeof(float);
    return prefill_split_workspace_full(B, T, H);
}

size_t prefill_split_workspace_min(int B, int T, int H)
{
    const size_t bh = (size_t)B * H;
    const size_t one = bh * kRec;
    const size_t full = prefill_split_workspace_full(B, T, H);
    return full <= one ? full : one + bh * kDK * kDV * sizeof(float);
}

namespace {

cudaError_t split_setup()
{
    cudaError_t e = cudaFuncSetAttribute(prefill_prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)PP_TOTAL);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(prefill_chain_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)CH_TOTAL);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(prefill_chain_t_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)TC_TOTAL);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(prefill_chain_t_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)TC_TOTAL);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(prefill_prep_scalar_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)PS_TOTAL);
    return e;
}

// A scalar gate (or none) with no fused steps before the path: the records come from
// prefill_prep_scalar_kernel, with the decays the per-head chain's kScalar form assumes.
bool scalar_records(const ForwardArgs &a) { return a.gate != KDA_GATE_CHANNEL && a.prep_flags == 0; }

cudaError_t rec_u_tensor_map(uint8_t *ws, size_t nrec, CUtensorMap *m);

// sms_free: the SMs the launch can expect to have (all of them unless a chain runs beside
// it), which sizes the persistent scalar-gate kernel's grid at two CTAs per SM.
// pdl: launched programmatically dependent on the kernel before it in the stream (a
// per-head chain), so that its CTAs are placed once the chain's are resident.
cudaError_t run_prep(const ForwardArgs &a, uint8_t *ws, int n0, int nb, cudaStream_t stream, int sms_free = 0,
                     bool pdl = false)
{
    const size_t bh = (size_t)a.B * a.H;
    CUtensorMap u_map;
    memset(&u_map, 0, sizeof(u_map));
    cudaError_t em = rec_u_tensor_map(ws, bh * (size_t)nb, &u_map);
    if (em != cudaSuccess) return em;
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    // the scalar-gate kernel is persistent, two CTAs per SM that can expect to be free;
    // the per-channel one takes one CTA per chunk (prefetching for the CTA half the SM
    // count further on: measured best among an eighth, a quarter, three eighths, a half,
    // one and two SM counts on the long-context shapes)
    const size_t nitems = bh * (size_t)nb;
    const size_t grid = std::min(nitems, (size_t)2 * (size_t)(sms_free > 0 ? std::min(sms_free, sms) : sms));
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kNT);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    const __nv_bfloat16 *qb = static_cast<const __nv_bfloat16 *>(a.q), *kb = static_cast<const __nv_bfloat16 *>(a.k),
                        *vb = static_cast<const __nv_bfloat16 *>(a.v);
    if (scalar_records(a)) {
        cfg.gridDim = dim3((unsigned)grid);
        cfg.dynamicSmemBytes = PS_TOTAL;
        e = cudaLaunchKernelEx(&cfg, prefill_prep_scalar_kernel, qb, kb, vb,
                               a.gate == KDA_GATE_SCALAR ? a.log_alpha : (const float *)nullptr, a.beta, ws, a.T, a.H,
                               n0, nb, (int)nitems, a.scale, u_map);
    } else {
        cfg.gridDim = dim3((unsigned)nitems);
        cfg.dynamicSmemBytes = PP_TOTAL;
        e = cudaLaunchKernelEx(&cfg, prefill_prep_kernel, qb, kb, vb, a.log_alpha, a.beta, ws, a.T, a.H, n0, nb,
                               a.scale, a.prep_flags, (int)a.gate, sms / 2, u_map);
    }
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e == cudaSuccess) note_launch();
    return e;
}

// cuTensorMapEncodeTiled from the driver, looked up once (the library links the CUDA
// runtime statically and not the driver library)
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
        else
            cudaGetLastError();
    });
    return fn;
}

// out [B, T, H, dv] fp32 as a 4-D tensor (dv, H, T, B), boxes of one head's 64 tokens:
// the per-head chain's output tile of one chunk.  The T axis has its own bound, so the
// ragged last chunk of a sequence writes no row of the next one.
cudaError_t out_tensor_map(const ForwardArgs &a, CUtensorMap *m)
{
    const PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc) return cudaErrorNotSupported;
    const cuuint64_t dims[4] = {(cuuint64_t)kDV, (cuuint64_t)a.H, (cuuint64_t)a.T, (cuuint64_t)a.B};
    const cuuint64_t strides[3] = {(cuuint64_t)kDV * 4u, (cuuint64_t)a.H * kDV * 4u, (cuuint64_t)a.T * a.H * kDV * 4u};
    const cuuint32_t box[4] = {(cuuint32_t)kDV, 1u, (cuuint32_t)kC, 1u};
    const cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
    const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, a.out, dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// The U rows of nrec consecutive records from ws as a 3-D tensor (32 floats, 256 rows of
// (slice, token), record), one box per record, 128-byte swizzle in shared memory.
cudaError_t rec_u_tensor_map(uint8_t *ws, size_t nrec, CUtensorMap *m)
{
    const PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc) return cudaErrorNotSupported;
    const cuuint64_t dims[3] = {(cuuint64_t)kDVS, (cuuint64_t)(kNSL * kC), (cuuint64_t)nrec};
    const cuuint64_t strides[2] = {(cuuint64_t)kDVS * 4u, (cuuint64_t)kRec};
    const cuuint32_t box[3] = {(cuuint32_t)kDVS, (cuuint32_t)(kNSL * kC), 1u};
    const cuuint32_t estr[3] = {1u, 1u, 1u};
    const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, ws + R_U, dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t run_chain(const ForwardArgs &a, bool per_head, const uint8_t *ws, int n0, int nb, const float *s_in,
                      float *s_out, int mode, const float *s_add, cudaStream_t stream)
{
    const size_t bh = (size_t)a.B * a.H;
    if (per_head) {
        CUtensorMap out_map;
        memset(&out_map, 0, sizeof(out_map));
        if (!(mode & kChainNoOut)) {
            const cudaError_t e = out_tensor_map(a, &out_map);
            if (e != cudaSuccess) return e;
        }
        if (scalar_records(a))
            prefill_chain_t_kernel<true><<<(unsigned)bh, kTThreads, TC_TOTAL, stream>>>(ws, s_in, s_out, out_map, a.T,
                                                                                     a.H, n0, nb, mode, s_add);
        else
            prefill_chain_t_kernel<false><<<(unsigned)bh, kTThreads, TC_TOTAL, stream>>>(ws, s_in, s_out, out_map,
                                                                                      a.T, a.H, n0, nb, mode, s_add);
    } else
        prefill_chain_kernel<<<(unsigned)(bh * kNSL), kChainThreads, CH_TOTAL, stream>>>(ws, s_in, s_out, a.out, a.T,
                                                                                     a.H, n0, nb, mode, s_add);
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) note_launch();
    return e;
}

// start = fold over the earlier segments: S = F_0; S = F_j + P_j S for j = 1..R-1.
// One CTA per (b, h, 32-column slice); P_j staged in shared memory with a padded
// row pitch; thread (row, half) owns 16 columns.  fp32.
constexpr int kAffPitch = 129;
constexpr uint32_t kAffSmem = (128 * kAffPitch + 128 * 32) * 4;

__global__ void __launch_bounds__(256, 1)
affine_compose_kernel(const float *__restrict__ P, const float *__restrict__ F, int R, int BH,
                      float *__restrict__ start)
{
    extern __shared__ __align__(16) float asmem[];
    float *sP = asmem;                      // [128][129]
    float *sS = asmem + 128 * kAffPitch;    // [128][32] current state slice
    const int tid = threadIdx.x;
    const int slice = blockIdx.x % kNSL, bh = blockIdx.x / kNSL;
    const int r = tid >> 1, c0 = 16 * (tid & 1);
    const size_t stride = (size_t)BH * kDK * kDV;
    const size_t base = ((size_t)bh * kDK + r) * kDV + kDVS * slice + c0;
#pragma unroll
    for (int j = 0; j < 16; ++j) sS[r * 32 + c0 + j] = F[base + j];
    for (int seg = 1; seg < R; ++seg) {
        const float *Pj = P + (size_t)seg * stride + (size_t)bh * kDK * kDK;
        __syncthreads();
        for (int id = tid; id < 128 * 128; id += 256) sP[(id >> 7) * kAffPitch + (id & 127)] = Pj[id];
        __syncthreads();
        float acc[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) acc[j] = F[(size_t)seg * stride + base + j];
        for (int c = 0; c < 128; ++c) {
            const float pv = sP[r * kAffPitch + c];
#pragma unroll
            for (int j = 0; j < 16; ++j) acc[j] += pv * sS[c * 32 + c0 + j];
        }
        __syncthreads();
#pragma unroll
        for (int j = 0; j < 16; ++j) sS[r * 32 + c0 + j] = acc[j];
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < 16; ++j) start[base + j] = sS[r * 32 + c0 + j];
}

}  // namespace

// The sequence is processed in blocks of L chunks, L as large as the workspace
// allows: prep over the block's chunks of every head, then the chain over them.
// When L < the number of chunks, the state between blocks is carried in the
// workspace after the records.
namespace {

// Blocks of up to L chunks, all on the caller's stream: prep(0), then chain(i) and prep(i + 1)
// for each block i.  prep(i + 1) is launched programmatically dependent on chain(i): it
// starts once every chain CTA is resident (the chain releases its dependents first thing),
// so its CTAs fill the SMs the chain leaves and never hold an SM a chain CTA is waiting
// for; it fills slot (i + 1) % 2 while chain(i) reads slot i % 2.  chain(i + 1), an
// ordinary launch, starts after everything before it in the stream has completed, so
// prep(i + 1) also follows chain(i - 1), the previous reader of its slot.  Neither
// kernel waits on the other inside a kernel.  (With the two kernels on two streams ordered
// by events, the chunk-local CTAs, dispatched at the same moment, often took every SM
// first: the chain of a block then started tens of microseconds late.)  The first and the
// last block are shorter (kPipeEndChunks), which shortens the stretches where only one of
// the kernels runs (the first prep, the last chain): B1 H32 T65536 3.74 -> 3.54 ms with
// end blocks of 32 chunks (16: 3.55, 8: 3.74); uniform blocks of 128 chunks measured
// slower, of 32 slower still.
constexpr int kPipeEndChunks = 32;

cudaError_t run_pipelined(const ForwardArgs &a, uint8_t *ws, int L, cudaStream_t stream)
{
    const int nchunks = (a.T + kC - 1) / kC;
    const size_t bh = (size_t)a.B * a.H;
    const size_t slot = bh * (size_t)L * kRec;
    float *carry = reinterpret_cast<float *>(ws + 2 * slot);
    const int E = min(L, kPipeEndChunks);
    auto block_len = [&](int n0) {
        const int rem = nchunks - n0;
        if (n0 == 0) return min(E, rem);
        if (rem <= E) return rem;
        return min(L, rem - E);
    };
    int nblk = 0;
    for (int n0 = 0; n0 < nchunks; n0 += block_len(n0)) ++nblk;
    const int sms = device_sms();
    const int sms_beside_chain = sms - (int)std::min<size_t>(bh, (size_t)sms / 2);
    cudaError_t e = run_prep(a, ws, 0, block_len(0), stream);
    int n0 = 0;
    for (int i = 0; i < nblk && e == cudaSuccess; ++i) {
        const int nb = block_len(n0);
        e = run_chain(a, true, ws + (size_t)(i & 1) * slot, n0, nb, i == 0 ? a.s0 : carry,
                      i == nblk - 1 ? a.sT : carry, 0, nullptr, stream);
        if (e == cudaSuccess && i + 1 < nblk) {
            const int n1 = n0 + nb;
            e = run_prep(a, ws + (size_t)((i + 1) & 1) * slot, n1, block_len(n1), stream, sms_beside_chain, true);
        }
        n0 += nb;
    }
    return e;
}

}  // namespace

cudaError_t launch_prefill_split(const ForwardArgs &a, uint8_t *ws, size_t ws_bytes, cudaStream_t stream, int T_whole)
{
    const int nchunks = (a.T + kC - 1) / kC;
    const size_t bh = (size_t)a.B * a.H;
    const size_t per_chunk = bh * kRec;
    const size_t state_bytes = bh * kDK * kDV * sizeof(float);
    const bool per_head = split_per_head(a.B, T_whole > 0 ? T_whole : a.T, a.H);
    cudaError_t e = split_setup();
    if (e != cudaSuccess) return e;
    if (per_head && pipelined_shape(bh, (size_t)nchunks, device_sms()) &&
        ws_bytes >= state_bytes + 2 * (size_t)kPipeMinChunks * per_chunk) {
        const size_t fit = (ws_bytes - state_bytes) / (2 * per_chunk);
        return run_pipelined(a, ws, (int)std::min<size_t>(fit, kPipeChunks), stream);
    }
    int L;
    if (ws_bytes >= per_chunk * (size_t)nchunks) {
        L = nchunks;
    } else {
        if (ws_bytes < per_chunk + state_bytes) return cudaErrorInvalidValue;
        L = (int)((ws_bytes - state_bytes) / per_chunk);
    }
    float *carry = (L < nchunks) ? reinterpret_cast<float *>(ws + per_chunk * (size_t)L) : nullptr;
    for (int n0 = 0; n0 < nchunks; n0 += L) {
        const int nb = min(L, nchunks - n0);
        e = run_prep(a, ws, n0, nb, stream);
        if (e != cudaSuccess) return e;
        const float *s_in = (n0 == 0) ? a.s0 : carry;
        float *s_out = (n0 + nb >= nchunks) ? a.sT : carry;
        e = run_chain(a, per_head, ws, n0, nb, s_in, s_out, 0, nullptr, stream);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

// Segment phases of a time-axis split: the whole segment is one block (the records
// stay in the workspace for the correction).
cudaError_t launch_segment_local(const ForwardArgs &a, float *transfer, uint8_t *ws, cudaStream_t stream)
{
    const int nchunks = (a.T + kC - 1) / kC;
    const bool per_head = (size_t)a.B * a.H * kNSL > (size_t)device_sms();
    cudaError_t e = split_setup();
    if (e == cudaSuccess) e = run_prep(a, ws, 0, nchunks, stream);
    // outputs and final state of the segment from the given start (zero if none)
    if (e == cudaSuccess) e = run_chain(a, per_head, ws, 0, nchunks, a.s0, a.sT, 0, nullptr, stream);
    // the segment's transfer: the state alone, propagated from S = I
    if (e == cudaSuccess)
        e = run_chain(a, per_head, ws, 0, nchunks, nullptr, transfer, kChainIdentityS0 | kChainZeroU | kChainNoOut,
                      nullptr, stream);
    return e;
}

cudaError_t launch_segment_correct(const ForwardArgs &a, const float *start, const float *local_final,
                                   const uint8_t *ws, cudaStream_t stream)
{
    const int nchunks = (a.T + kC - 1) / kC;
    const bool per_head = (size_t)a.B * a.H * kNSL > (size_t)device_sms();
    cudaError_t e = split_setup();
    // out += outputs of the start state propagated alone; final = local final + that state
    if (e == cudaSuccess)
        e = run_chain(a, per_head, ws, 0, nchunks, start, a.sT, kChainZeroU | kChainAccumOut, local_final, stream);
    return e;
}

cudaError_t launch_affine_compose(const float *transfers, const float *local_finals, int R, int BH, float *start,
                                  cudaStream_t stream)
{
    cudaError_t e = cudaFuncSetAttribute(affine_compose_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kAffSmem);
    if (e != cudaSuccess) return e;
    affine_compose_kernel<<<(unsigned)((size_t)BH * kNSL), 256, kAffSmem, stream>>>(transfers, local_finals, R, BH,
                                                                                   start);
    e = cudaGetLastError();
    if (e == cudaSuccess) note_launch();
    return e;
}

cudaError_t launch_selftest_timeout(unsigned int wait_ms, cudaStream_t stream)
{
    int dev = 0, khz = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&khz, cudaDevAttrClockRate, dev);
    if (e != cudaSuccess) return e;
    selftest_timeout_kernel<<<1, 32, 0, stream>>>((long long)wait_ms * (long long)khz);
    e = cudaGetLastError();
    if (e == cudaSuccess) note_launch();
    return e;
}

cudaError_t take_split_device_status(unsigned int *status)
{
    unsigned int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbol(status, g_split_device_status, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    if (*status) e = cudaMemcpyToSymbol(g_split_device_status, &zero, sizeof(unsigned int));
    return e;
}

}  // namespace kda
