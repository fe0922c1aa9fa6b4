/*
 * attn_bwd.cuh -- fused attention backward pass for sm_100a.
 *
 * The pages name the backward pass only through the statistics the forward
 * pass saves so that it can recompute instead of storing the N x N matrices
 * ("science-depth-m4-047", section 3, point (c)).  Given the forward inputs, O,
 * the upstream gradient dO and the saved LSE, with s_ij = scale q_i . k_j:
 *     P_ij  = exp(s_ij - LSE_i)              (recomputed, masked j > i if causal)
 *     dV_j  = sum_i P_ij dO_i
 *     dP_ij = dO_i . v_j
 *     dS_ij = P_ij (dP_ij - D_i),   D_i = sum_c dO_ic O_ic  (= sum_j P_ij dP_ij)
 *     dQ_i  = scale sum_j dS_ij k_j,   dK_j = scale sum_i dS_ij q_i
 * No N x N matrix reaches device memory.
 *
 * bwd_pre_kernel   D_i and LSE_i * log2(e) into row-padded workspace arrays; zero
 *                  the fp32 dQ accumulator.
 * bwd_main_kernel  one CTA per (head, 128-row K/V block j), looping over the Q
 *                  blocks i that see block j.  K_j and V_j stay in shared memory;
 *                  Q_i and dO_i stream through a 2-stage TMA ring.  Per i, on
 *                  the tensor cores (TMEM accumulators):
 *                      S^T  = K_j Q_i^T   -> TMEM A      dP^T = V_j dO_i^T -> TMEM B
 *                  warps 0-3 (thread = K/V row = TMEM lane) turn them into P^T
 *                  (bf16, over TMEM A) and scale * dS^T (bf16, over TMEM B, and
 *                  into shared memory as dS), then
 *                      dV_j += P^T dO_i  (A from TMEM)    dK_j += dS^T Q_i  (A from TMEM)
 *                      dQ_i partial = dS K_j  (A, B from shared memory) -> TMEM A
 *                  and warps 4-7 add the dQ partial into the fp32 accumulator
 *                  with vector atomics.  At the end warps 4-7 write dK_j, dV_j.
 * bwd_post_kernel  dQ accumulator -> bf16.
 */

constexpr int BWD_THREADS = 320;    // warps 0-3 dS, 4-7 dQ readout + epilogue, 8 TMA, 9 MMA
constexpr int BWD_LOAD_WARP = 8;
constexpr int BWD_MMA_WARP = 9;

struct BwdParams {
    __nv_bfloat16* dq;
    __nv_bfloat16* dk;
    __nv_bfloat16* dv;
    float* dq_acc;       // [BH, N, D] fp32
    const float* Dp;     // [BH, Np]  D_i, zero-padded
    const float* lse2;   // [BH, Np]  LSE_i * log2(e), zero-padded
    int N, Np, BH, nblk;
    float scale;         // multiplies q.k
    float scale_log2;    // scale * log2(e)
    uint64_t wait_limit_ns;
};

template <int D>
struct BwdCfg {
    static constexpr uint32_t TILE = BLOCK_M * D * 2;
    static constexpr int CHUNKS = D / CHUNK_ELEMS;
    static constexpr uint32_t K_OFF = 0, V_OFF = TILE;
    static constexpr uint32_t Q_OFF = 2 * TILE;                 // [2] stages
    static constexpr uint32_t DO_OFF = 4 * TILE;                // [2] stages
    static constexpr uint32_t DS_OFF = 6 * TILE;                // 128 x 128 bf16 = 32 KB
    static constexpr uint32_t BAR_OFF = DS_OFF + 32768;
    static constexpr int NUM_BARS = 1 + 4 + 6;
    static constexpr uint32_t MISC_OFF = BAR_OFF + 8 * NUM_BARS;
    static constexpr int SMEM_BYTES = MISC_OFF + 16 + 1024;
    static constexpr uint32_t RA = 0, RB = 128, DV_COL = 256, DK_COL = 256 + D;
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
};

__host__ __device__ constexpr uint32_t idesc_bf16_ab(int M, int N, bool a_mn, bool b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) |
           ((b_mn ? 1u : 0u) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
           (static_cast<uint32_t>(M >> 4) << 24);
}

/* D_i = dO_i . O_i, lse2_i = LSE_i log2(e) (zero past N), dq_acc = 0.
 * One warp per padded row. */
template <int D>
__global__ void __launch_bounds__(256)
bwd_pre_kernel(const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ dout,
               const float* __restrict__ lse, float* __restrict__ Dp, float* __restrict__ lse2,
               float* __restrict__ dq_acc, int N, int Np, int BH) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t prow = static_cast<int64_t>(blockIdx.x) * 8 + warp;     // over BH * Np
    if (prow >= static_cast<int64_t>(BH) * Np) return;
    const int bh = static_cast<int>(prow / Np), i = static_cast<int>(prow % Np);
    float dsum = 0.0f;
    if (i < N) {
        const int64_t base = (static_cast<int64_t>(bh) * N + i) * D;
#pragma unroll
        for (int c = lane; c < D; c += 32) {
            dsum += __bfloat162float(o[base + c]) * __bfloat162float(dout[base + c]);
            dq_acc[base + c] = 0.0f;
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, off);
    if (lane == 0) {
        Dp[prow] = i < N ? dsum : 0.0f;
        lse2[prow] = i < N ? lse[static_cast<int64_t>(bh) * N + i] * LOG2E : 0.0f;
    }
}

__global__ void bwd_post_kernel(const float* __restrict__ acc, __nv_bfloat16* __restrict__ dq,
                                int64_t n) {
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x)
        dq[i] = __float2bfloat16_rn(acc[i]);
}

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(BWD_THREADS, 1)
bwd_main_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                const BwdParams p) {
    using C = BwdCfg<D>;
    constexpr uint32_t TILE = C::TILE;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* const base_ptr = smem_raw + (base - raw);
    const uint32_t sK = base + C::K_OFF, sV = base + C::V_OFF, sDS = base + C::DS_OFF;
    const uint32_t bars = base + C::BAR_OFF;
    const uint32_t bar_kv = bars;
    auto bar_full = [&](int s) { return bars + 8 + 8u * s; };
    auto bar_empty = [&](int s) { return bars + 24 + 8u * s; };
    const uint32_t bar_s = bars + 40, bar_p = bars + 48, bar_dq = bars + 56, bar_dqf = bars + 64;
    const uint32_t bar_dkv = bars + 72, bar_drain = bars + 80;
    uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + C::MISC_OFF);
    volatile uint32_t* const abort_flag = reinterpret_cast<volatile uint32_t*>(base_ptr + C::MISC_OFF + 4);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint64_t wlim = p.wait_limit_ns;
    const int jb = blockIdx.x, bh = blockIdx.y;
    const int ib0 = CAUSAL ? jb : 0;
    const int nq = p.nblk - ib0;                 // Q blocks that see this K/V block

    if (threadIdx.x == 0) {
        mbar_init(bar_kv, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar_full(s), 1);
            mbar_init(bar_empty(s), 1);
        }
        mbar_init(bar_s, 1);
        mbar_init(bar_p, BLOCK_M);
        mbar_init(bar_dq, 1);
        mbar_init(bar_dqf, BLOCK_M);
        mbar_init(bar_dkv, 1);
        mbar_init(bar_drain, 1);
        *abort_flag = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == BWD_MMA_WARP) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(tmem_slot)), "r"(TMEM_COLS) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == BWD_LOAD_WARP) {
        /* ---------------- TMA: K_j, V_j once; Q_i, dO_i per Q block ---------------- */
        if (lane == 0) {
            mbar_arrive_expect_tx(bar_kv, 2 * TILE);
            for (int c = 0; c < C::CHUNKS; ++c) {
                tma_load_3d(&tm_k, sK + c * CHUNK_BYTES, bar_kv, c * CHUNK_ELEMS, jb * BLOCK_M, bh);
                tma_load_3d(&tm_v, sV + c * CHUNK_BYTES, bar_kv, c * CHUNK_ELEMS, jb * BLOCK_M, bh);
            }
            int issued = 0;
            for (int it = 0; it < nq; ++it) {
                const int s = it & 1;
                if (!mbar_wait(bar_empty(s), ((it >> 1) & 1) ^ 1, abort_flag, wlim)) break;
                const int ib = ib0 + it;
                mbar_arrive_expect_tx(bar_full(s), 2 * TILE);
                for (int c = 0; c < C::CHUNKS; ++c) {
                    tma_load_3d(&tm_q, base + C::Q_OFF + s * TILE + c * CHUNK_BYTES, bar_full(s),
                                c * CHUNK_ELEMS, ib * BLOCK_M, bh);
                    tma_load_3d(&tm_do, base + C::DO_OFF + s * TILE + c * CHUNK_BYTES, bar_full(s),
                                c * CHUNK_ELEMS, ib * BLOCK_M, bh);
                }
                ++issued;
            }
            // every copy this thread issued lands before the CTA can exit
            mbar_drain_wait(bar_kv, 0, wlim);
            const int back = issued < 2 ? issued : 2;
            for (int b = 1; b <= back; ++b) {
                const int it = issued - b;
                mbar_drain_wait(bar_full(it & 1), (it >> 1) & 1, wlim);
            }
        }
        __syncwarp();
    } else if (warp == BWD_MMA_WARP) {
        /* ---------------- MMA issue ---------------- */
        if (lane == 0) {
            constexpr uint32_t ID_KQ = idesc_bf16_ab(BLOCK_M, BLOCK_M, false, false);  // S^T, dP^T
            constexpr uint32_t ID_ACC = idesc_bf16_ab(BLOCK_M, D, false, true);        // dV, dK
            constexpr uint32_t ID_DQ = idesc_bf16_ab(BLOCK_M, D, true, true);          // dQ
            const uint32_t ta = tmem + C::RA, tb = tmem + C::RB;
            const uint32_t tdv = tmem + C::DV_COL, tdk = tmem + C::DK_COL;
            const uint64_t kd = sdesc_sw128(sK, 16, 1024);                  // K-major
            const uint64_t vd = sdesc_sw128(sV, 16, 1024);                  // K-major
            const uint64_t k_mn = sdesc_sw128(sK, CHUNK_BYTES, 1024);       // K_j as MN-major B
            const uint64_t ds_mn = sdesc_sw128(sDS, 16384, 1024);           // dS as MN-major A
            bool ok = mbar_wait(bar_kv, 0, abort_flag, wlim);
            for (int it = 0; it < nq && ok; ++it) {
                const int s = it & 1;
                ok = mbar_wait(bar_full(s), (it >> 1) & 1, abort_flag, wlim);
                if (!ok) break;
                if (it > 0) {
                    // the dQ partial of the previous block has been read out of TMEM A
                    ok = mbar_wait(bar_dqf, (it - 1) & 1, abort_flag, wlim);
                    if (!ok) break;
                    tc_fence_after();
                }
                const uint32_t sq = base + C::Q_OFF + s * TILE, sdo = base + C::DO_OFF + s * TILE;
                issue_qk<D>(ta, kd, sdesc_sw128(sq, 16, 1024), ID_KQ);          // S^T = K Q^T
                issue_qk<D>(tb, vd, sdesc_sw128(sdo, 16, 1024), ID_KQ);         // dP^T = V dO^T
                mma_commit(bar_s);
                ok = mbar_wait(bar_p, it & 1, abort_flag, wlim);
                if (!ok) break;
                tc_fence_after();
                const uint64_t do_mn = sdesc_sw128(sdo, CHUNK_BYTES, 1024);
                const uint64_t q_mn = sdesc_sw128(sq, CHUNK_BYTES, 1024);
#pragma unroll
                for (int kk = 0; kk < BLOCK_M / 16; ++kk) {
                    const uint64_t off = static_cast<uint64_t>((kk * 16 * 128) >> 4);
                    const uint32_t acc = (it > 0 || kk > 0) ? 1u : 0u;
                    mma_ts(tdv, ta + kk * 8, do_mn + off, ID_ACC, acc);         // dV += P^T dO
                    mma_ts(tdk, tb + kk * 8, q_mn + off, ID_ACC, acc);          // dK += dS^T Q
                }
#pragma unroll
                for (int kk = 0; kk < BLOCK_M / 16; ++kk) {
                    const uint64_t off = static_cast<uint64_t>((kk * 16 * 128) >> 4);
                    mma_ss(ta, ds_mn + off, k_mn + off, ID_DQ, kk > 0 ? 1u : 0u);  // dQ = dS K
                }
                mma_commit(bar_dq);
                mma_commit(bar_empty(s));
            }
            if (ok) mma_commit(bar_dkv);
            mma_commit(bar_drain);
            mbar_drain_wait(bar_drain, 0, wlim);
        }
        __syncwarp();
    } else if (warp < 4) {
        /* ---------------- P^T and dS^T, thread = K/V row (TMEM lane) ---------------- */
        const int r = warp * 32 + lane;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
        const float c = p.scale_log2, sc = p.scale;
        const int kv = jb * BLOCK_M + r;
        for (int it = 0; it < nq; ++it) {
            const int ib = ib0 + it;
            bool ok = mbar_wait(bar_s, it & 1, abort_flag, wlim);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            const float* lse2 = p.lse2 + static_cast<int64_t>(bh) * p.Np + ib * BLOCK_M;
            const float* dvec = p.Dp + static_cast<int64_t>(bh) * p.Np + ib * BLOCK_M;
            const bool diag = CAUSAL && ib == jb;
#pragma unroll 1
            for (int ch = 0; ch < BLOCK_M / 32; ++ch) {
                uint32_t sv[32], dpv[32];
                tmem_ld32_wait(lane_base + C::RA + ch * 32, sv);
                tmem_ld32_wait(lane_base + C::RB + ch * 32, dpv);
                uint32_t pk[16], dk[16];
#pragma unroll
                for (int e = 0; e < 32; e += 4) {
                    const float4 l4 = __ldg(reinterpret_cast<const float4*>(lse2 + ch * 32 + e));
                    const float4 d4 = __ldg(reinterpret_cast<const float4*>(dvec + ch * 32 + e));
                    const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
                    const float dvv[4] = {d4.x, d4.y, d4.z, d4.w};
                    float pp[4], dd[4];
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        const int ql = ch * 32 + e + h;
                        float pv = ex2(fmaf(__uint_as_float(sv[e + h]), c, -lv[h]));
                        if (diag && ql < r) pv = 0.0f;        // key kv row r masked for query ql < r
                        pp[h] = pv;
                        dd[h] = pv * (__uint_as_float(dpv[e + h]) - dvv[h]) * sc;
                    }
                    pk[e / 2] = pack_bf16(pp[0], pp[1]);
                    pk[e / 2 + 1] = pack_bf16(pp[2], pp[3]);
                    dk[e / 2] = pack_bf16(dd[0], dd[1]);
                    dk[e / 2 + 1] = pack_bf16(dd[2], dd[3]);
                }
                tmem_st16(lane_base + C::RA + ch * 16, pk);
                tmem_st16(lane_base + C::RB + ch * 16, dk);
                // dS into shared memory as the MN-major A operand of dQ = dS K:
                // query index contiguous in 64-wide atoms (16 KB apart), K/V row r
                // at 128 B, 8-row groups 1 KB apart, 16-byte units swizzled by r % 8
                const uint32_t atom = sDS + (ch >> 1) * 16384 + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int unit = (ch & 1) * 4 + u;
                    const uint32_t addr = atom + ((unit ^ (r & 7)) << 4);
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr),
                                 "r"(dk[4 * u]), "r"(dk[4 * u + 1]), "r"(dk[4 * u + 2]),
                                 "r"(dk[4 * u + 3]) : "memory");
                }
            }
            (void)kv;
            tmem_wait_st();
            tc_fence_before();
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // dS visible to the MMA
            mbar_arrive(bar_p);
        }
    } else if (warp < 8) {
        /* ---------------- dQ readout (thread = query row) and the dK, dV epilogue ---------------- */
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
        bool ok = true;
        for (int it = 0; it < nq; ++it) {
            const int ib = ib0 + it;
            ok = mbar_wait(bar_dq, it & 1, abort_flag, wlim);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            const int row = ib * BLOCK_M + r;
            float* dst = p.dq_acc + (static_cast<int64_t>(bh) * p.N + (row < p.N ? row : 0)) * D;
#pragma unroll
            for (int ch = 0; ch < D / 32; ++ch) {
                uint32_t v[32];
                tmem_ld32_wait(lane_base + C::RA + ch * 32, v);
                if (row < p.N) {
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        atomicAdd(reinterpret_cast<float4*>(dst + ch * 32 + 4 * e),
                                  make_float4(__uint_as_float(v[4 * e]), __uint_as_float(v[4 * e + 1]),
                                              __uint_as_float(v[4 * e + 2]),
                                              __uint_as_float(v[4 * e + 3])));
                }
            }
            tc_fence_before();
            mbar_arrive(bar_dqf);
        }
        if (ok) {
            ok = mbar_wait(bar_dkv, 0, abort_flag, wlim);
            ok = __all_sync(0xffffffffu, ok);
        }
        if (ok) {
            tc_fence_after();
            const int kvrow = jb * BLOCK_M + r;
            const int64_t off = (static_cast<int64_t>(bh) * p.N + (kvrow < p.N ? kvrow : 0)) * D;
#pragma unroll
            for (int which = 0; which < 2; ++which) {
                __nv_bfloat16* out = (which ? p.dk : p.dv) + off;
                const uint32_t col = which ? C::DK_COL : C::DV_COL;
#pragma unroll
                for (int ch = 0; ch < D / 32; ++ch) {
                    uint32_t v[32];
                    tmem_ld32_wait(lane_base + col + ch * 32, v);
                    if (kvrow < p.N) {
                        uint4* d4 = reinterpret_cast<uint4*>(out + ch * 32);
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            d4[e] = make_uint4(
                                pack_bf16(__uint_as_float(v[8 * e]), __uint_as_float(v[8 * e + 1])),
                                pack_bf16(__uint_as_float(v[8 * e + 2]), __uint_as_float(v[8 * e + 3])),
                                pack_bf16(__uint_as_float(v[8 * e + 4]), __uint_as_float(v[8 * e + 5])),
                                pack_bf16(__uint_as_float(v[8 * e + 6]), __uint_as_float(v[8 * e + 7])));
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == BWD_MMA_WARP) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(TMEM_COLS) : "memory");
    }
}
