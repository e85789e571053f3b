// Chunk-local kernel of the two-kernel prefill for the scalar-gate members of the
// family (Gated DeltaNet: one decay per token and head; DeltaNet: none), bf16 inputs,
// dk = dv = 128.  Included by kda_prefill_split.cu inside its namespace: it writes the
// same chunk record as prefill_prep_kernel, read by the same chain kernels.
//
// With one decay per token every factor of the chunk algebra is a per-token scalar
// ("Kimi Delta Attention: The Linear Attention Behind Kimi K2 and Qwen3", §DeltaNet,
// Gated DeltaNet, and KDA, comparison table: a scalar alpha_t instead of Diag(alpha_t)),
// so the decay factors out of the contractions.  With G_t the in-chunk inclusive sum of
// log alpha (G non-increasing, G <= 0):
//
//   [K; Q] K^T            exact bf16 inputs: one tensor-core term
//   A_ij = beta_i e^{G_i - G_j} (k_i . k_j)         (j < i),  every factor <= 1
//   M_ij = scale e^{G_i - G_j} (q_i . k_j)          (j <= i)
//   R = (I + A)^-1 Diag(beta)
//   Wr = (R Diag(e^G)) K,  U = R V                   K and V exact: two terms each
//   Qr = scale Diag(e^G) Q,  Kb = Diag(e^{G_last - G}) K
//
// which is the record of the per-channel kernel with the reference point m = 0:
// e^m = e^{G_last - m} = 1 and e^{G_last} in every channel.  No factor exceeds 1.
// Exponentials are per token, not per pair: e^{G_i - G_j} = a_i b_j with
// a = e^{G - G_ref}, b = e^{G_ref - G} and G_ref midway between the chunk's extremes of
// G; a chunk whose range of G exceeds 2 kScalarGMax (a factor could overflow) takes
// e^{G_i - G_j} pair by pair instead.

// shared memory (bytes); tiles in the no-swizzle canonical layout of kda_tc_ptx.cuh
constexpr uint32_t PS_K = 0;              // K rows: K-major (outer token, inner dk); the B of P1, MN-major B of Wr
constexpr uint32_t PS_Q = 16384;          // Q rows: rows 64..127 of the [K; Q] A tile of P1
constexpr uint32_t PS_V = 98304;          // V: MN-major B of U
constexpr uint32_t PS_BETA = 114688;      // fp32 [64]
constexpr uint32_t PS_G = PS_BETA + 256;  // fp32 [64]: log alpha, then G, then e^G (after the readout)
constexpr uint32_t PS_B = PS_G + 256;     // fp32 [64]: b = e^{G_ref - G}
constexpr uint32_t PS_REF = PS_B + 256;   // fp32 G_ref; int wide
constexpr uint32_t PS_MBAR = PS_REF + 16;
constexpr uint32_t PS_TMEMP = PS_MBAR + 8;
constexpr uint32_t PS_TOTAL = PS_TMEMP + 8;
static_assert(PS_TOTAL <= 115712, "two CTAs per SM");
// after P1 (the [K; Q] tile's Q rows are free): the solve's A and T (fp32, row pitch
// kPitch), then R: [R Diag(e^G) hi | lo | R hi | lo], 8 KB each (K-major, outer row,
// inner token).  Qr, Kb and M go to the record straight from registers.
constexpr uint32_t PS_AMAT = 16384, PS_TMAT = PS_AMAT + 64 * kPitch * 4;
constexpr uint32_t PS_R = PS_TMAT + 64 * kPitch * 4;
static_assert(PS_R + 32768 <= PS_V, "R tiles below V");
// after P2: U staged for its tensor store (Wr goes to the record from registers)
constexpr uint32_t PS_U = 49152;
static_assert(PS_U + 32768 <= PS_V, "U below V");
constexpr float kScalarGMax = 80.f;       // largest |G - G_ref| of the factored form (e^80 < 2^127)

// Persistent: CTA x takes the work items x, x + gridDim.x, ... of the launch, and the
// inputs of its next chunk land while it finishes the
// current one: the Q rows once the solve has released their space, K, V, the decays and
// beta once the second product has read them.
__global__ void __launch_bounds__(kNT, 2)
prefill_prep_scalar_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                           const __nv_bfloat16 *__restrict__ v, const float *__restrict__ log_alpha,
                           const float *__restrict__ beta, uint8_t *__restrict__ ws, int T, int H, int n0, int nb,
                           int nitems, float scale, const __grid_constant__ CUtensorMap u_map)
{
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t sbase = (uint32_t)__cvta_generic_to_shared(smem);
    float *sBeta = reinterpret_cast<float *>(smem + PS_BETA);
    float *sG = reinterpret_cast<float *>(smem + PS_G);
    float *sB = reinterpret_cast<float *>(smem + PS_B);
    const uint32_t mbar = sbase + PS_MBAR;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int lrow = 32 * (warp & 3) + lane;          // tensor-memory lane of the readouts
    const int half = warp >> 2;
    // work item -> chunk: items take the block's chunks from the last to the first, every
    // (b, h) of a chunk together, so the chunks the chain reads first are written last and
    // are still in L2 when it starts.  Record index bh * nb + local chunk; first token and
    // length of the chunk; row(item, t) = its token t's row in [B, T, H]
    const int nbh = nitems / nb;
    auto item_bh = [&](int item) { return item % nbh; };
    auto item_loc = [&](int item) { return nb - 1 - item / nbh; };
    auto rec_index = [&](int item) { return item_bh(item) * nb + item_loc(item); };
    auto chunk_t0 = [&](int item) { return (n0 + item_loc(item)) * kC; };
    auto chunk_len = [&](int item) { return min(kC, T - chunk_t0(item)); };
    auto row = [&](int item, int t) {
        const int bh = item_bh(item);
        return ((size_t)(bh / H) * T + chunk_t0(item) + t) * H + bh % H;
    };
    // input loads of chunk `item` (rows past the chunk's end zero-filled): eight
    // consecutive threads take the eight rows of one core matrix, so a warp's 16-byte
    // pieces fill 512 contiguous bytes of the tile (no bank conflicts)
    auto load_rows = [&](int item, const __nv_bfloat16 *src, uint32_t dst, int d) {
        const int c = chunk_len(item);
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int id = tid + kNT * r, t = (id & 7) | ((id >> 7) << 3), g = (id >> 3) & 15;
            const bool okt = t < c;
            cp_async16(sbase + dst + core_off(t, 8 * g, RW_SO, RW_SI), src + row(item, okt ? t : 0) * d + 8 * g,
                       okt ? 16u : 0u);
        }
    };
    auto load_scalars = [&](int item) {
        if (tid < kC) {
            const bool okt = tid < chunk_len(item);
            const size_t r = row(item, okt ? tid : 0);
            if (log_alpha) cp_async4(sbase + PS_G + 4u * tid, log_alpha + r, okt ? 4u : 0u);
            else sG[tid] = 0.f;
            cp_async4(sbase + PS_BETA + 4u * tid, beta + r, okt ? 4u : 0u);
        }
    };

    int item = blockIdx.x;
    if (item >= nitems) return;
    load_rows(item, q, PS_Q, kDK);
    load_rows(item, k, PS_K, kDK);
    load_rows(item, v, PS_V, kDV);
    load_scalars(item);
    cp_async_commit();
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     :: "r"(sbase + PS_TMEMP), "r"(TMP_COLS) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (tid == 0) {
        mbar_init(mbar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + PS_TMEMP);
    const uint32_t tlane = (uint32_t)(32 * (warp & 3)) << 16;
    float *Am = reinterpret_cast<float *>(smem + PS_AMAT);
    float *Tm = reinterpret_cast<float *>(smem + PS_TMAT);
    bool failed = false;

    for (; item < nitems; item += gridDim.x) {
        const int next = item + (int)gridDim.x;
        uint8_t *rec = ws + (size_t)rec_index(item) * kRec;
        // ---- this chunk's inputs have landed (and every read of the previous chunk's
        // tensor memory is done)
        cp_async_wait_all();
        proxy_fence();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        // ---- P1: [K; Q] K^T on the exact inputs; rows 0..63 -> A, rows 64..127 -> M
        if (tid == 0) {
            mma_split(tmem + TMP_AM, sbase + PS_K, 0u, RW_SI, RW_SO, sbase + PS_K, 0u, RW_SI, RW_SO, kDK / 16,
                      idesc_bf16(128, 64, 0, 0), false, false, false);
            umma_commit(mbar);
        }
        // ---- in-chunk inclusive sums of the decay (warp 0; padded tokens add 0)
        if (warp == 0) {
            float a0 = sG[lane], a1 = sG[lane + 32];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float u0 = __shfl_up_sync(0xffffffffu, a0, o);
                const float u1 = __shfl_up_sync(0xffffffffu, a1, o);
                if (lane >= o) { a0 += u0; a1 += u1; }
            }
            a1 += __shfl_sync(0xffffffffu, a0, 31);
            sG[lane] = a0;
            sG[lane + 32] = a1;
            float mx = fmaxf(a0, a1), mn = fminf(a0, a1);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
            }
            const float gref = 0.5f * (mx + mn);
            const bool wide = !(mx - mn <= 2.f * kScalarGMax);
            sB[lane] = wide ? 0.f : __expf(gref - a0);
            sB[lane + 32] = wide ? 0.f : __expf(gref - a1);
            if (lane == 0) {
                reinterpret_cast<float *>(smem + PS_REF)[0] = gref;
                reinterpret_cast<int *>(smem + PS_REF)[1] = wide ? 1 : 0;
            }
        }
        __syncthreads();
        const float g_last = sG[kC - 1];
        const float gref = reinterpret_cast<const float *>(smem + PS_REF)[0];
        const bool wide = reinterpret_cast<const int *>(smem + PS_REF)[1] != 0;
        // the record's per-channel decays with m = 0: e^m = 1, e^{G_last}, e^{G_last - m} = 1
        if (tid < kDK) {
            reinterpret_cast<float *>(rec + R_EM)[tid] = 1.f;
            reinterpret_cast<float *>(rec + R_GAM)[tid] = __expf(g_last);
            reinterpret_cast<float *>(rec + R_EL)[tid] = 1.f;
        }
        // ---- Qr = scale e^G q and Kb = e^{G_last - G} k, split, straight to the record:
        // thread (warp w, lane l) takes token 8 w + l % 8 and channel groups l / 8 + 4 r, so
        // a warp's 16-byte pieces fill 512 contiguous bytes (of the tiles in shared memory
        // and of the record) and a thread needs one token's factors
        {
            const int tq = (lane & 7) + 8 * warp;
            const float gt = sG[tq];
            const float fq = scale * __expf(gt), fk = __expf(g_last - gt);
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int g = (lane >> 3) + 4 * r;
                const uint32_t o = core_off(tq, 8 * g, RW_SO, RW_SI);
                const uint4 qv = *reinterpret_cast<const uint4 *>(smem + PS_Q + o);
                const uint4 kv = *reinterpret_cast<const uint4 *>(smem + PS_K + o);
                const __nv_bfloat16 *qb = reinterpret_cast<const __nv_bfloat16 *>(&qv);
                const __nv_bfloat16 *kb = reinterpret_cast<const __nv_bfloat16 *>(&kv);
                float y[8];
                uint4 hv, lv;
#pragma unroll
                for (int i = 0; i < 8; ++i) y[i] = fq * __bfloat162float(qb[i]);
                split8(y, hv, lv);
                *reinterpret_cast<uint4 *>(rec + R_WQ + 16384u + o) = hv;
                *reinterpret_cast<uint4 *>(rec + R_WQ_LO + 16384u + o) = lv;
#pragma unroll
                for (int i = 0; i < 8; ++i) y[i] = fk * __bfloat162float(kb[i]);
                split8(y, hv, lv);
                *reinterpret_cast<uint4 *>(rec + R_KT + o) = hv;
                *reinterpret_cast<uint4 *>(rec + R_KT_LO + o) = lv;
            }
        }
        const bool p1_done = mbar_wait(mbar, 0u);
        if (tid == 0) bulk_wait_read();      // the previous chunk's U store has read its staging
        if ((failed = __syncthreads_or(!p1_done) != 0)) break;

        // ---- A = Diag(beta) strictly_lower(...) to shared memory, M to the record
        {
            tc_fence_after();
            float x[32];
            tmem_ld16(tmem + tlane + TMP_AM + 32 * half, *reinterpret_cast<float (*)[16]>(x));
            tmem_ld16(tmem + tlane + TMP_AM + 32 * half + 16, *reinterpret_cast<float (*)[16]>(x + 16));
            const int i = lrow & 63;
            const float gi = sG[i];
            const float ai = wide ? 0.f : __expf(gi - gref);
            // e^{G_i - G_j}: a_i b_j, or pair by pair in a wide chunk
            auto fac = [&](int j) { return wide ? __expf(gi - sG[j]) : ai * sB[j]; };
            if (lrow < 64) {
                const float bi = sBeta[i];
#pragma unroll
                for (int e4 = 0; e4 < 8; ++e4) {
                    float y[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int j = 32 * half + 4 * e4 + e;
                        y[e] = (j < i) ? bi * fac(j) * x[4 * e4 + e] : 0.f;
                    }
                    *reinterpret_cast<float4 *>(Am + i * kPitch + 32 * half + 4 * e4) =
                        make_float4(y[0], y[1], y[2], y[3]);
                }
            } else {
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    float y[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int j = 32 * half + 8 * g + e;
                        y[e] = (j <= i) ? scale * fac(j) * x[8 * g + e] : 0.f;
                    }
                    const uint32_t o = core_off(i, 32 * half + 8 * g, H_SO, H_SI);
                    uint4 hv, lv;
                    split8(y, hv, lv);
                    *reinterpret_cast<uint4 *>(rec + R_M + o) = hv;
                    *reinterpret_cast<uint4 *>(rec + R_M_LO + o) = lv;
                }
            }
        }
        __syncthreads();

        // ---- T = (I + A)^-1; R = T Diag(beta) and R Diag(e^G), split, as the A of P2
        if (tid >= kNT - kC) sG[tid - (kNT - kC)] = __expf(sG[tid - (kNT - kC)]);   // G is read no more: e^G
        unit_lower_inverse(Am, Tm, tid);
        __syncthreads();
        // A is free: the next chunk's Q rows land where it was
        if (next < nitems) {
            load_rows(next, q, PS_Q, kDK);
            cp_async_commit();
        }
        for (int id = tid; id < 512; id += kNT) {
            const int i = id >> 3, jg = id & 7;
            const float4 t0v = *reinterpret_cast<const float4 *>(Tm + i * kPitch + 8 * jg);
            const float4 t1v = *reinterpret_cast<const float4 *>(Tm + i * kPitch + 8 * jg + 4);
            const float *bj = sBeta + 8 * jg;
            const float *egj = sG + 8 * jg;
            float y[8] = {t0v.x * bj[0], t0v.y * bj[1], t0v.z * bj[2], t0v.w * bj[3],
                          t1v.x * bj[4], t1v.y * bj[5], t1v.z * bj[6], t1v.w * bj[7]};
            const uint32_t o = core_off(i, 8 * jg, H_SO, H_SI);
            st_split8(smem, PS_R + 16384u + o, PS_R + 24576u + o, y);              // R
#pragma unroll
            for (int e = 0; e < 8; ++e) y[e] *= egj[e];
            st_split8(smem, PS_R + o, PS_R + 8192u + o, y);                        // R Diag(e^G)
        }
        proxy_fence();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            // [R e^G; .] K (K rows read MN-major as B): rows 0..63 are Wr;
            // [. ; R] V (the tile viewed from R e^G lo, so rows 64..127 are R): rows 64..127
            // are U.  K and V are exact bf16: two terms each
            mma_split(tmem + TMP_W, sbase + PS_R, sbase + PS_R + 8192u, H_SI, H_SO,
                      sbase + PS_K, 0u, RW_SO, RW_SI, kC / 16, idesc_bf16(128, kDK, 0, 1), false, true, false);
            mma_split(tmem + TMP_U, sbase + PS_R + 8192u, sbase + PS_R + 16384u, H_SI, H_SO,
                      sbase + PS_V, 0u, RW_SO, RW_SI, kC / 16, idesc_bf16(128, kDV, 0, 1), false, true, false);
            umma_commit(mbar);
        }
        if ((failed = __syncthreads_or(!mbar_wait(mbar, 1u)) != 0)) break;
        tc_fence_after();
        // K, V, the decays and beta are read: the next chunk's land in their place
        if (next < nitems) {
            load_rows(next, k, PS_K, kDK);
            load_rows(next, v, PS_V, kDV);
            load_scalars(next);
            cp_async_commit();
        }
        if (lrow < 64) {
            // Wr: lane = row i, 64 key channels per thread, straight to the record
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
                    const uint32_t o = core_off(lrow, c0 + 8 * g, RW_SO, RW_SI);
                    uint4 hv, lv;
                    split8(y, hv, lv);
                    *reinterpret_cast<uint4 *>(rec + R_WQ + o) = hv;
                    *reinterpret_cast<uint4 *>(rec + R_WQ_LO + o) = lv;
                }
            }
        } else {
            // U: lane 64 + token, 64 value columns per thread = two slices, staged as the
            // swizzled rows of the tensor store's box
#pragma unroll
            for (int s2 = 0; s2 < 2; ++s2) {
                const int r = (2 * half + s2) * kC + lrow - 64;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    float x[16];
                    tmem_ld16(tmem + tlane + TMP_U + 64 * half + 32 * s2 + 16 * hh, x);
#pragma unroll
                    for (int g = 0; g < 4; ++g)
                        *reinterpret_cast<float4 *>(smem + PS_U + u_stage_off(r, 4 * hh + g)) =
                            make_float4(x[4 * g], x[4 * g + 1], x[4 * g + 2], x[4 * g + 3]);
                }
            }
        }
        proxy_fence();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tma_store_3d(&u_map, sbase + PS_U, 0, 0, rec_index(item));
            bulk_commit();
        }
    }

    if (failed && tid == 0) atomicOr(&g_split_device_status, 1u);
    cp_async_wait_all();                     // loads in flight land before shared memory goes
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem), "r"(TMP_COLS) : "memory");
    }
    if (tid == 0) bulk_wait_read();          // shared memory stays until the copies have read it
}
