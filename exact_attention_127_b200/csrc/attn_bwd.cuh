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
 * bwd_pre_kernel   D_i and LSE_i * log2(e) into row-padded workspace arrays (the
 *                  host zeroes the fp32 dQ accumulator before it).
 * bwd_main_kernel  one CTA per (head, 128-row K/V block j), looping over the Q
 *                  blocks i that see block j; CTAs start longest first within
 *                  groups of heads.  K_j and V_j stay in shared memory;
 *                  Q_i and dO_i stream through a TMA ring (2 stages at d = 128,
 *                  4 at d = 64).  Per i, on the tensor cores (TMEM accumulators):
 *                      S^T  = K_j Q_i^T   -> TMEM A      dP^T = V_j dO_i^T -> TMEM B
 *                  warps 0-7 (thread = K/V row = TMEM lane; warps w and w+4 share
 *                  the lanes and split the 128 queries in halves) turn S^T into
 *                  P^T (bf16, packed over the first half of its own columns of
 *                  TMEM A); then, while they form scale * dS (bf16) into shared
 *                  memory once dP^T is there,
 *                      dV_j += P^T dO_i               (A from TMEM)
 *                      S^T of block i+1               (overwrites P^T: MMAs run in issue order)
 *                  and once dS is stored
 *                      dQ_i partial = dS K_j          (A, B from shared memory) -> TMEM dQ
 *                      dK_j += dS^T Q_i               (A, B from shared memory)
 *                  At d = 128 the dQ partial lies over dP^T, whose columns the next
 *                  block's dP^T needs: warps 12-15 (thread = query row) take it out
 *                  of TMEM as soon as it lands, staging a quarter over dO_i (which
 *                  dV_i and dP^T_i have read) and holding the rest in registers,
 *                  and release the columns; the second half of the partial follows
 *                  the first through the dO_i half, so the Q_i half of the stage
 *                  goes back as soon as dK_i has read it and the next Q block's
 *                  load waits for no reduce.  At d = 64 (own columns) they stage
 *                  it over the freed Q_i / dO_i stage.  One of them adds the staged halves into the
 *                  fp32 accumulator with TMA bulk reduce-adds, while warps 0-7
 *                  already work on block i+1.  At the end warps 0-7 write dK_j, dV_j.
 *                  Warp 8 issues the TMA loads, warp 9 the MMAs; setmaxnreg
 *                  gives the P/dS warps the registers of the others.
 * bwd_post_kernel  dQ accumulator -> bf16.
 *
 * The dQ accumulator is tiled [BH][Q block][D/4][128 rows][4], so a Q block's
 * partial is one contiguous 128 x D fp32 region: two bulk reduce-adds of its
 * halves, staged in the same layout in shared memory.
 */

constexpr int BWD_HEAD_GROUP = 8;   // heads per group of the grid order (bwd_main_kernel)
constexpr int BWD_THREADS = 512;    // warps 0-7 P, dS, epilogue; 8 TMA; 9 MMA; 12-15 dQ readout
constexpr int BWD_COMPUTE = 256;
constexpr int BWD_LOAD_WARP = 8;
constexpr int BWD_MMA_WARP = 9;
constexpr int BWD_READ_WARP0 = 12;
constexpr int BWD_READERS = 128;
/* Register split (setmaxnreg) of the 512 x 128 registers the launch holds:
 * the P/dS warpgroups rise to 168, the TMA/MMA warpgroup (with the two warps
 * that have no role) drops to 56 and the readout warpgroup to 120 (96 columns
 * of the dQ partial held at once: with 512 threads ptxas allows no instruction
 * more than 128 live registers). */
constexpr int BWD_LAUNCH_REGS = 128;  // per thread at launch (checked on the host before launching)
constexpr int BWD_COMPUTE_REGS = 168;
constexpr int BWD_CTRL_REGS = 56;
constexpr int BWD_READ_REGS = 120;
static_assert(2 * 128 * BWD_COMPUTE_REGS + 128 * BWD_CTRL_REGS + 128 * BWD_READ_REGS ==
                  BWD_THREADS * BWD_LAUNCH_REGS,
              "register split");

struct BwdParams {
    __nv_bfloat16* dq;
    __nv_bfloat16* dk;
    __nv_bfloat16* dv;
    float* dq_acc;       // [BH, Np/128, D/4, 128, 4] fp32
    const float* Dp;     // [BH, Np]  D_i, zero-padded
    const float* lse2;   // [BH, Np]  LSE_i * log2(e), zero-padded
    int N, Np, BH, nblk;
    float scale;         // multiplies q.k
    float scale_log2;    // scale * log2(e)
    uint64_t wait_limit_ns;
    int withhold;        // test hook: the TMA warp loads nothing, so every wait runs out
};

template <int D>
struct BwdCfg {
    static constexpr uint32_t TILE = BLOCK_M * D * 2;
    static constexpr int CHUNKS = D / CHUNK_ELEMS;
    static constexpr uint32_t K_OFF = 0, V_OFF = TILE;
    // Q_i / dO_i ring: 2 stages at D = 128 (shared memory is full), 4 at D = 64,
    // where the load of Q block i+2 then need not wait for block i's dQ partial
    // to leave the stage it is staged in
    static constexpr int QS = D == 64 ? 4 : 2;
    static constexpr uint32_t Q_OFF = 2 * TILE;                 // [QS] stages
    static constexpr uint32_t DO_OFF = Q_OFF + QS * TILE;       // [QS] stages
    static constexpr uint32_t DS_OFF = DO_OFF + QS * TILE;      // 128 x 128 bf16 = 32 KB
    static constexpr uint32_t BAR_OFF = DS_OFF + 32768;
    static constexpr int NUM_BARS = 12 + 5 * QS;
    static constexpr uint32_t MISC_OFF = BAR_OFF + 8 * NUM_BARS;
    static constexpr int SMEM_BYTES = MISC_OFF + 16 + 1024;
    // TMEM columns: S^T / P^T, dP^T, the dV and dK accumulators, the dQ partial
    // (over dP^T when no columns are left, i.e. at D = 128)
    static constexpr uint32_t RA = 0, RB = 128, DV_COL = 256, DK_COL = 256 + D;
    static constexpr uint32_t DQ_COL = (256 + 2 * D + D <= 512) ? 256 + 2 * D : RB;
    static constexpr bool DQ_OVER_DP = DQ_COL == RB;
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
};

__host__ __device__ constexpr uint32_t idesc_bf16_ab(int M, int N, bool a_mn, bool b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) |
           ((b_mn ? 1u : 0u) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
           (static_cast<uint32_t>(M >> 4) << 24);
}

/* TMEM column of the packed P^T columns for queries [16 kk, 16 kk + 16): the
 * half h = kk / 4 of the queries is packed at the start of its own 64 columns. */
__device__ __forceinline__ uint32_t bwd_p_col(int kk) {
    return static_cast<uint32_t>((kk >> 2) * 64 + (kk & 3) * 8);
}

/* D_i = dO_i . O_i, lse2_i = LSE_i log2(e) (zero past N).  D / 8 threads per
 * padded row, each with one 16-byte load of O_i and of dO_i (every pointer is
 * 16-byte aligned, checked on the host), so a warp reads whole rows; the
 * partial sums of a row meet through shuffles among its lanes. */
constexpr int BWD_PRE_THREADS = 256;
template <int D>
__global__ void __launch_bounds__(BWD_PRE_THREADS)
bwd_pre_kernel(const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ dout,
               const float* __restrict__ lse, float* __restrict__ Dp, float* __restrict__ lse2,
               int N, int Np, int BH) {
    constexpr int TPR = D / 8;                       // threads per row
    constexpr int ROWS = BWD_PRE_THREADS / TPR;      // rows per block
    const int part = threadIdx.x % TPR;
    const int64_t prow = static_cast<int64_t>(blockIdx.x) * ROWS + threadIdx.x / TPR;  // over BH * Np
    const bool valid = prow < static_cast<int64_t>(BH) * Np;   // the same for a row's lanes
    int bh = 0, i = 0;
    float dsum = 0.0f;
    if (valid) {
        bh = static_cast<int>(prow / Np);
        i = static_cast<int>(prow % Np);
        if (i < N) {
            const int64_t off = (static_cast<int64_t>(bh) * N + i) * D + part * 8;
            const uint4 a = __ldg(reinterpret_cast<const uint4*>(o + off));
            const uint4 g = __ldg(reinterpret_cast<const uint4*>(dout + off));
            const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, gw[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 af = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&aw[e]));
                const float2 gf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&gw[e]));
                dsum += af.x * gf.x;
                dsum += af.y * gf.y;
            }
        }
    }
#pragma unroll
    for (int off = TPR / 2; off > 0; off >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, off);
    if (valid && part == 0) {
        Dp[prow] = i < N ? dsum : 0.0f;
        lse2[prow] = i < N ? lse[static_cast<int64_t>(bh) * N + i] * LOG2E : 0.0f;
    }
}

/* Tiled fp32 dQ accumulator -> bf16 [BH, N, D].  One CTA per (head, Q block):
 * coalesced reads of the tile, a transpose through shared memory, and a
 * contiguous copy of the block's rows. */
template <int D>
__global__ void __launch_bounds__(BLOCK_M)
bwd_post_kernel(const float* __restrict__ acc, __nv_bfloat16* __restrict__ dq, int N, int nblk) {
    constexpr int ROW = D + 8;                   // padded bf16 row: fewer bank conflicts
    __shared__ __align__(16) __nv_bfloat16 tile[BLOCK_M * ROW];
    const int t = threadIdx.x;
    const int bh = blockIdx.x / nblk, ib = blockIdx.x % nblk;
    const float4* src = reinterpret_cast<const float4*>(acc) +
                        static_cast<int64_t>(blockIdx.x) * (D / 4) * BLOCK_M;
#pragma unroll 4
    for (int g = 0; g < D / 4; ++g) {
        const float4 v = src[g * BLOCK_M + t];
        *reinterpret_cast<uint2*>(&tile[t * ROW + 4 * g]) =
            make_uint2(pack_bf16(v.x, v.y), pack_bf16(v.z, v.w));
    }
    __syncthreads();
    const int rows = min(BLOCK_M, N - ib * BLOCK_M);
    uint4* dst = reinterpret_cast<uint4*>(dq + (static_cast<int64_t>(bh) * N + ib * BLOCK_M) * D);
    for (int i = t; i < rows * (D / 8); i += BLOCK_M) {
        const int row = i / (D / 8), c16 = i % (D / 8);
        dst[i] = *reinterpret_cast<const uint4*>(&tile[row * ROW + c16 * 8]);
    }
}

/* dQ_i partial = dS K_j: A = dS (MN-major, shared memory), B = K_j (MN-major). */
__device__ __forceinline__ void bwd_issue_dq(uint32_t tdq, uint64_t ds_mn, uint64_t k_mn, uint32_t idesc) {
#pragma unroll 1
    for (int kk = 0; kk < BLOCK_M / 16; ++kk) {
        const uint64_t off = static_cast<uint64_t>((kk * 16 * 128) >> 4);
        mma_ss(tdq, ds_mn + off, k_mn + off, idesc, kk > 0 ? 1u : 0u);
    }
}

/* dV_j += P^T dO_i: A = P^T (TMEM), B = dO_i (MN-major). */
__device__ __forceinline__ void bwd_issue_dv(uint32_t tdv, uint32_t ta, uint64_t do_mn, uint32_t idesc,
                                             bool accumulate) {
#pragma unroll 1
    for (int kk = 0; kk < BLOCK_M / 16; ++kk) {
        const uint64_t off = static_cast<uint64_t>((kk * 16 * 128) >> 4);
        mma_ts(tdv, ta + bwd_p_col(kk), do_mn + off, idesc, (accumulate || kk > 0) ? 1u : 0u);
    }
}

/* Elementwise product of two f32 pairs (mul.rn.f32x2). */
__device__ __forceinline__ uint64_t bwd_fmul2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

/* fp32 add of `bytes` bytes of shared memory at src into global memory at dst
 * by the TMA engine (both 16-byte aligned, bytes a multiple of 16). */
__device__ __forceinline__ void bulk_reduce_add_f32(float* dst, uint32_t src, uint32_t bytes) {
    asm volatile("cp.reduce.async.bulk.global.shared::cta.bulk_group.add.f32 [%0], [%1], %2;"
                 ::"l"(reinterpret_cast<uint64_t>(dst)), "r"(src), "r"(bytes) : "memory");
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
    const uint32_t bar_s = bars + 8, bar_p = bars + 16, bar_pt = bars + 24, bar_dqf = bars + 32;
    const uint32_t bar_dkv = bars + 40, bar_drain = bars + 48, bar_dp = bars + 56;
    const uint32_t bar_rd_q = bars + 64;                            // first half of the dQ tile staged
    const uint32_t bar_rd_do = bars + 72;                           // second half staged
    const uint32_t bar_dq = bars + 80;                              // the dQ partial is in TMEM
    const uint32_t bar_sdo = bars + 88;                             // dO half read by the first reduce
    // Per ring stage.  Q_i and dO_i of a stage land, and are handed back,
    // separately: the readout stages the first half of the dQ partial over Q_i
    // and reduce-adds it first, so the next Q block can load while the second
    // half (over dO_i) is staged.
    constexpr int QS = C::QS;
    auto bar_full_q = [&](int s) { return bars + 96 + 8u * s; };
    auto bar_full_do = [&](int s) { return bars + 96 + 8u * (QS + s); };
    auto bar_empty = [&](int s) { return bars + 96 + 8u * (2 * QS + s); };    // dK_i has read Q_i
    auto bar_free_q = [&](int s) { return bars + 96 + 8u * (3 * QS + s); };   // Q half handed back
    auto bar_free_do = [&](int s) { return bars + 96 + 8u * (4 * QS + s); };  // dO half handed back
    uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + C::MISC_OFF);
    volatile uint32_t* const abort_flag = reinterpret_cast<volatile uint32_t*>(base_ptr + C::MISC_OFF + 4);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint64_t wlim = p.wait_limit_ns;
    // Grid order: groups of BWD_HEAD_GROUP heads, and within a group every head's
    // K/V block 0 first, then block 1, ...  The hardware starts CTAs in index
    // order, so for causal masks (block j has nblk - j Q blocks) the longest
    // CTAs start first and the end of the launch is made of short ones; a group's
    // Q, dO, K, V stay within L2 while its CTAs run.
    int jb, bh;
    {
        const int per_group = BWD_HEAD_GROUP * p.nblk;
        const int g = blockIdx.x / per_group, r = blockIdx.x - g * per_group;
        const int heads = min(BWD_HEAD_GROUP, p.BH - g * BWD_HEAD_GROUP);
        jb = r / heads;
        bh = g * BWD_HEAD_GROUP + (r - jb * heads);
    }
    const int ib0 = CAUSAL ? jb : 0;
    const int nq = p.nblk - ib0;                 // Q blocks that see this K/V block

    if (threadIdx.x == 0) {
        mbar_init(bar_kv, 1);
        for (int s = 0; s < QS; ++s) {
            mbar_init(bar_full_q(s), 1);
            mbar_init(bar_full_do(s), 1);
            mbar_init(bar_empty(s), 1);
            mbar_init(bar_free_q(s), 1);
            mbar_init(bar_free_do(s), 1);
        }
        mbar_init(bar_rd_q, BWD_READERS);
        mbar_init(bar_rd_do, BWD_READERS);
        mbar_init(bar_s, 1);
        mbar_init(bar_dp, 1);
        mbar_init(bar_dq, 1);
        mbar_init(bar_sdo, 1);
        mbar_init(bar_p, BWD_COMPUTE);
        mbar_init(bar_pt, BWD_COMPUTE);
        mbar_init(bar_dqf, BWD_READERS);
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
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(BWD_CTRL_REGS) : "memory");
        /* ---------------- TMA: K_j, V_j once; Q_i, dO_i per Q block ---------------- */
        if (lane == 0 && !p.withhold) {
            mbar_arrive_expect_tx(bar_kv, 2 * TILE);
            for (int c = 0; c < C::CHUNKS; ++c) {
                tma_load_3d(&tm_k, sK + c * CHUNK_BYTES, bar_kv, c * CHUNK_ELEMS, jb * BLOCK_M, bh);
                tma_load_3d(&tm_v, sV + c * CHUNK_BYTES, bar_kv, c * CHUNK_ELEMS, jb * BLOCK_M, bh);
            }
            int issued_q = 0, issued_do = 0;
            for (int it = 0; it < nq; ++it) {
                const int s = it % QS;
                const uint32_t use = static_cast<uint32_t>(it / QS);
                const int ib = ib0 + it;
                if (!mbar_wait_inl(bar_free_q(s), (use & 1u) ^ 1u, abort_flag, wlim)) break;
                mbar_arrive_expect_tx(bar_full_q(s), TILE);
                for (int c = 0; c < C::CHUNKS; ++c)
                    tma_load_3d(&tm_q, base + C::Q_OFF + s * TILE + c * CHUNK_BYTES, bar_full_q(s),
                                c * CHUNK_ELEMS, ib * BLOCK_M, bh);
                ++issued_q;
                if (!mbar_wait_inl(bar_free_do(s), (use & 1u) ^ 1u, abort_flag, wlim)) break;
                mbar_arrive_expect_tx(bar_full_do(s), TILE);
                for (int c = 0; c < C::CHUNKS; ++c)
                    tma_load_3d(&tm_do, base + C::DO_OFF + s * TILE + c * CHUNK_BYTES, bar_full_do(s),
                                c * CHUNK_ELEMS, ib * BLOCK_M, bh);
                ++issued_do;
            }
            // every copy this thread issued lands before the CTA can exit
            mbar_drain_wait_inl(bar_kv, 0, wlim);
            for (int b = 1; b <= (issued_q < QS ? issued_q : QS); ++b) {
                const int it = issued_q - b;
                mbar_drain_wait_inl(bar_full_q(it % QS), (it / QS) & 1, wlim);
            }
            for (int b = 1; b <= (issued_do < QS ? issued_do : QS); ++b) {
                const int it = issued_do - b;
                mbar_drain_wait_inl(bar_full_do(it % QS), (it / QS) & 1, wlim);
            }
        }
        __syncwarp();
    } else if (warp == BWD_MMA_WARP) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(BWD_CTRL_REGS) : "memory");
        /* ---------------- MMA issue ---------------- */
        if (lane == 0) {
            constexpr uint32_t ID_KQ = idesc_bf16_ab(BLOCK_M, BLOCK_M, false, false);  // S^T, dP^T
            constexpr uint32_t ID_ACC = idesc_bf16_ab(BLOCK_M, D, false, true);        // dV, dK
            constexpr uint32_t ID_DQ = idesc_bf16_ab(BLOCK_M, D, true, true);          // dQ
            const uint32_t ta = tmem + C::RA, tb = tmem + C::RB;
            const uint32_t tdv = tmem + C::DV_COL, tdk = tmem + C::DK_COL, tdq = tmem + C::DQ_COL;
            const uint64_t kd = sdesc_sw128(sK, 16, 1024);                  // K-major
            const uint64_t vd = sdesc_sw128(sV, 16, 1024);                  // K-major
            const uint64_t k_mn = sdesc_sw128(sK, CHUNK_BYTES, 1024);       // K_j as MN-major B
            const uint64_t ds_mn = sdesc_sw128(sDS, 16384, 1024);           // dS as MN-major A (dQ)
            const uint64_t ds_k = sdesc_sw128(sDS, 16, 1024);               // dS^T as K-major A (dK)
            bool ok = mbar_wait_inl(bar_kv, 0, abort_flag, wlim);
            if (ok) ok = mbar_wait_inl(bar_full_q(0), 0, abort_flag, wlim);
            if (ok) {
                tc_fence_after();
                issue_qk<D>(ta, kd, sdesc_sw128(base + C::Q_OFF, 16, 1024), ID_KQ);  // S^T = K Q^T
                mma_commit(bar_s);
            }
            for (int it = 0; it < nq && ok; ++it) {
                const int s = it % QS;
                const uint32_t sq = base + C::Q_OFF + s * TILE, sdo = base + C::DO_OFF + s * TILE;
                if (C::DQ_OVER_DP && it > 0) {
                    // dP^T overwrites the previous dQ partial: wait until it was read out
                    ok = mbar_wait_inl(bar_dqf, (it - 1) & 1, abort_flag, wlim);
                    if (!ok) break;
                    tc_fence_after();
                }
                ok = mbar_wait_inl(bar_full_do(s), (it / QS) & 1, abort_flag, wlim);   // dO_i landed
                if (!ok) break;
                issue_qk<D>(tb, vd, sdesc_sw128(sdo, 16, 1024), ID_KQ);         // dP^T = V dO^T
                mma_commit(bar_dp);
                const uint64_t do_mn = sdesc_sw128(sdo, CHUNK_BYTES, 1024);
                const uint64_t q_mn = sdesc_sw128(sq, CHUNK_BYTES, 1024);
                // the next S^T over P^T: the tensor core reads P^T for dV first
                auto issue_next_s = [&]() -> bool {
                    if (it + 1 >= nq) return true;
                    const int s1 = (it + 1) % QS;
                    if (!mbar_wait_inl(bar_full_q(s1), ((it + 1) / QS) & 1, abort_flag, wlim)) return false;
                    tc_fence_after();
                    issue_qk<D>(ta, kd, sdesc_sw128(base + C::Q_OFF + s1 * TILE, 16, 1024), ID_KQ);
                    mma_commit(bar_s);
                    return true;
                };
                // dV_i and the next S^T as soon as P^T is in TMEM, while warps 0-7
                // still form dS; then dQ_i and dK_i once dS is in shared memory
                ok = mbar_wait_inl(bar_pt, it & 1, abort_flag, wlim);        // P^T in TMEM
                if (!ok) break;
                tc_fence_after();
                bwd_issue_dv(tdv, ta, do_mn, ID_ACC, it > 0);
                ok = issue_next_s();
                if (!ok) break;
                ok = mbar_wait_inl(bar_p, it & 1, abort_flag, wlim);         // dS in shared memory
                if (!ok) break;
                tc_fence_after();
                if (!C::DQ_OVER_DP && it > 0) {
                    // the previous dQ partial has its own columns: read out yet?
                    ok = mbar_wait_inl(bar_dqf, (it - 1) & 1, abort_flag, wlim);
                    if (!ok) break;
                    tc_fence_after();
                }
                bwd_issue_dq(tdq, ds_mn, k_mn, ID_DQ);
                if constexpr (C::DQ_OVER_DP) mma_commit(bar_dq);   // the readout may take it now
#pragma unroll 1
                for (int kk = 0; kk < BLOCK_M / 16; ++kk) {
                    const uint64_t off_mn = static_cast<uint64_t>((kk * 16 * 128) >> 4);
                    const uint64_t off_k = static_cast<uint64_t>(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
                    mma_ss(tdk, ds_k + off_k, q_mn + off_mn, ID_ACC,
                           (it > 0 || kk > 0) ? 1u : 0u);                         // dK += dS^T Q
                }
                mma_commit(bar_empty(s));
            }
            if (ok) mma_commit(bar_dkv);
            mma_commit(bar_drain);
            mbar_drain_wait_inl(bar_drain, 0, wlim);
        }
        __syncwarp();
    } else if (warp >= BWD_READ_WARP0) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(BWD_READ_REGS) : "memory");
        /* ---------------- warps 12-15: the dQ partial of Q block i ----------------
         * Thread r = query row copies its row of the partial from TMEM into the
         * Q_i / dO_i stage, laid out as the accumulator tile, and releases the dQ
         * columns; at D = 128 early, as described below.  One thread adds each half
         * into the fp32 accumulator with a TMA bulk reduce-add as soon as it is
         * staged, and hands that half of the stage back to the producer once the
         * reduce has read it: no atomics through the SM's load/store path. */
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
        const bool leader = threadIdx.x == BWD_READ_WARP0 * 32;
        for (int it = 0; it < nq; ++it) {
            const int s = it % QS, ib = ib0 + it;
            if constexpr (C::DQ_OVER_DP) {
                /* dQ_i has landed over dP^T_i.  dV_i and dP^T_i, issued before it, have
                 * read dO_i, so the first half of the partial goes over dO_i at once and
                 * is reduce-added; the second half is held in registers meanwhile, the
                 * dQ columns (the next dP^T) are released, and it follows through the
                 * dO_i half once the first reduce has read it. */
                bool ok = mbar_wait_inl(bar_dq, it & 1, abort_flag, wlim);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                tc_fence_after();
                const uint32_t sq = base + C::Q_OFF + s * TILE, sdo = base + C::DO_OFF + s * TILE;
                float* tile = p.dq_acc + (static_cast<int64_t>(bh) * p.nblk + ib) * (BLOCK_M * D);
                // chunk 0 goes over dO_i first; chunks 1-3 (96 columns, as many as a thread
                // of this warpgroup holds) are then read and the columns released
                {
                    uint32_t v[32];
                    tmem_ld32_wait(lane_base + C::DQ_COL, v);
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const uint32_t dst = sdo + (e * BLOCK_M + r) * 16;
                        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(v[4 * e]),
                                     "r"(v[4 * e + 1]), "r"(v[4 * e + 2]), "r"(v[4 * e + 3]) : "memory");
                    }
                }
                uint32_t hv[96];
#pragma unroll
                for (int ch = 0; ch < 3; ++ch)
                    tmem_ld32_wait(lane_base + C::DQ_COL + 32 + ch * 32, hv + 32 * ch);
                tc_fence_before();
                mbar_arrive(bar_dqf);                 // every column read
#pragma unroll
                for (int e = 0; e < 8; ++e) {         // chunk 1: the rest of the dO_i half
                    const uint32_t dst = sdo + ((8 + e) * BLOCK_M + r) * 16;
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(hv[4 * e]),
                                 "r"(hv[4 * e + 1]), "r"(hv[4 * e + 2]), "r"(hv[4 * e + 3]) : "memory");
                }
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                mbar_arrive(bar_rd_do);
                // the Q_i half of the stage is not staged into: it goes back once dK_i
                // has read it; the second half of the partial follows the first through
                // the dO_i half once the first reduce has read it
                if (leader) {
                    if (mbar_wait_inl(bar_rd_do, it & 1, abort_flag, wlim)) {
                        bulk_reduce_add_f32(tile, sdo, TILE);
                        asm volatile("cp.async.bulk.commit_group;" ::: "memory");
                    }
                    if (mbar_wait_inl(bar_empty(s), (it / QS) & 1, abort_flag, wlim))   // dK_i done
                        mbar_arrive(bar_free_q(s));
                    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");   // first half read
                    mbar_arrive(bar_sdo);
                }
                ok = mbar_wait_inl(bar_sdo, it & 1, abort_flag, wlim);            // dO_i half free again
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
#pragma unroll
                for (int g = 0; g < D / 8; ++g) {
                    const uint32_t dst = sdo + (g * BLOCK_M + r) * 16;
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(hv[32 + 4 * g]),
                                 "r"(hv[32 + 4 * g + 1]), "r"(hv[32 + 4 * g + 2]), "r"(hv[32 + 4 * g + 3]) : "memory");
                }
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                mbar_arrive(bar_rd_q);
                if (leader && mbar_wait_inl(bar_rd_q, it & 1, abort_flag, wlim)) {
                    bulk_reduce_add_f32(tile + TILE / 4, sdo, TILE);
                    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
                    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");   // second half read
                    mbar_arrive(bar_free_do(s));
                }
                continue;
            }
            // D = 64: once dK_i has read Q_i, half 0 (column groups [0, D/8)) over Q_i,
            // half 1 over dO_i, each reduce-added as soon as it is staged
            bool ok = mbar_wait_inl(bar_empty(s), (it / QS) & 1, abort_flag, wlim);   // dK_i done
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            const uint32_t sq = base + C::Q_OFF + s * TILE, sdo = base + C::DO_OFF + s * TILE;
            float* tile = p.dq_acc + (static_cast<int64_t>(bh) * p.nblk + ib) * (BLOCK_M * D);
#pragma unroll 1
            for (int half = 0; half < 2 && ok; ++half) {
                const uint32_t dst0 = half ? sdo : sq;
#pragma unroll 1
                for (int ch = half * (D / 64); ch < (half + 1) * (D / 64); ++ch) {
                    uint32_t v[32];
                    tmem_ld32_wait(lane_base + C::DQ_COL + ch * 32, v);
                    if (ch == D / 32 - 1) {          // every column read: release them
                        tc_fence_before();
                        mbar_arrive(bar_dqf);
                    }
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int g = ch * 8 + e;     // float4 column group of the tile
                        const uint32_t dst = dst0 + ((g % (D / 8)) * BLOCK_M + r) * 16;
                        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(v[4 * e]),
                                     "r"(v[4 * e + 1]), "r"(v[4 * e + 2]), "r"(v[4 * e + 3]) : "memory");
                    }
                }
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // visible to the TMA
                const uint32_t bar_rd = half ? bar_rd_do : bar_rd_q;
                mbar_arrive(bar_rd);
                if (leader) {
                    if (!mbar_wait_inl(bar_rd, it & 1, abort_flag, wlim)) { ok = false; break; }
                    bulk_reduce_add_f32(tile + half * (TILE / 4), dst0, TILE);
                    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
                    // each half of the stage goes back as soon as its reduce has read it
                    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
                    mbar_arrive(half ? bar_free_do(s) : bar_free_q(s));
                }
            }
            if (!ok) break;
        }
        if (leader) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");   // reduces complete
    } else if (warp >= 8) {
        /* warps 10, 11: no role; their registers go to the P/dS warpgroups */
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(BWD_CTRL_REGS) : "memory");
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(BWD_COMPUTE_REGS) : "memory");
        /* ---------------- warps 0-7: P^T, dS, dK/dV epilogue ----------------
         * thread = TMEM lane = K/V row r; warp w covers lanes 32 (w % 4) .. and
         * the half h = w / 4 of the queries. */
        const int quarter = warp & 3, h = warp >> 2;
        const int r = quarter * 32 + lane;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
        const float c = p.scale_log2, sc = p.scale;
        const uint64_t c2 = f2pack(c, c), sc2 = f2pack(sc, sc);
        bool ok = true;
        for (int it = 0; it < nq; ++it) {
            const int ib = ib0 + it;
            const int64_t row0 = static_cast<int64_t>(bh) * p.Np + ib * BLOCK_M + 64 * h;
            const float* lse2 = p.lse2 + row0;
            const float* dvec = p.Dp + row0;
            // at D = 64 the LSE values of this half go out before the wait for S^T,
            // which hides their latency (an L2 round trip under the dQ reduce-adds); at
            // D = 128 the P/dS warps are not what the step waits for, and loading early
            // measured slower there
            constexpr int EARLY = D == 64 ? 16 : 0;
            float4 l4e[16];
#pragma unroll
            for (int e = 0; e < EARLY; ++e) l4e[e] = __ldg(reinterpret_cast<const float4*>(lse2) + e);
            ok = mbar_wait_inl(bar_s, it & 1, abort_flag, wlim);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            if (lane < 4 && it + 1 < nq) {
                // the next Q block's LSE and D values (two 128-byte lines each) into L1
                // now, so that their first reads next step do not wait on L2
                const float* nx = (lane < 2 ? lse2 : dvec) + BLOCK_M + 32 * (lane & 1);
                asm volatile("prefetch.global.L1 [%0];" ::"l"(nx));
            }
            // on the diagonal block key r is masked for the queries before it:
            // column ch * 32 + e of this half is masked when it is < mask_lim
            const bool diag = CAUSAL && ib == jb;
            const int mask_lim = diag ? r - 64 * h : 0;
            float pf[64];
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {
                uint32_t sv[32];
                tmem_ld32_wait(lane_base + C::RA + 64 * h + 32 * ch, sv);
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 32; e += 4) {
                    const float4 l4 = EARLY ? l4e[ch * 8 + e / 4]
                                            : __ldg(reinterpret_cast<const float4*>(lse2 + ch * 32 + e));
                    // c s - lse2 on pairs (f32x2: the same rounding as scalar fmaf)
                    float x[4];
                    f2unpack(ffma2(f2pack(__uint_as_float(sv[e]), __uint_as_float(sv[e + 1])), c2,
                                   f2pack(-l4.x, -l4.y)), x[0], x[1]);
                    f2unpack(ffma2(f2pack(__uint_as_float(sv[e + 2]), __uint_as_float(sv[e + 3])), c2,
                                   f2pack(-l4.z, -l4.w)), x[2], x[3]);
#pragma unroll
                    for (int hh = 0; hh < 4; ++hh) pf[ch * 32 + e + hh] = ex2(x[hh]);
                    if (diag) {   // warp-uniform: only the diagonal block masks
#pragma unroll
                        for (int hh = 0; hh < 4; ++hh)
                            if (ch * 32 + e + hh < mask_lim) pf[ch * 32 + e + hh] = 0.0f;
                    }
                    pk[e / 2] = pack_bf16(pf[ch * 32 + e], pf[ch * 32 + e + 1]);
                    pk[e / 2 + 1] = pack_bf16(pf[ch * 32 + e + 2], pf[ch * 32 + e + 3]);
                }
                tmem_st16(lane_base + C::RA + 64 * h + 16 * ch, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar_pt);    // P^T is in TMEM: dV and the next S^T may go
            float4 d4e[16];         // likewise the D values before the wait for dP^T
#pragma unroll
            for (int e = 0; e < EARLY; ++e) d4e[e] = __ldg(reinterpret_cast<const float4*>(dvec) + e);
            ok = mbar_wait_inl(bar_dp, it & 1, abort_flag, wlim);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            // dS into shared memory: 64-query atoms 16 KB apart, K/V row r at 128 B,
            // 8-row groups 1 KB apart, 16-byte units swizzled by r % 8 -- the MN-major
            // A operand of dQ = dS K and the K-major A operand of dK = dS^T Q
            const uint32_t atom = sDS + h * 16384 + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {
                uint32_t dpv[32];
                tmem_ld32_wait(lane_base + C::RB + 64 * h + 32 * ch, dpv);
                uint32_t dk[16];
#pragma unroll
                for (int e = 0; e < 32; e += 4) {
                    const float4 d4 = EARLY ? d4e[ch * 8 + e / 4]
                                            : __ldg(reinterpret_cast<const float4*>(dvec + ch * 32 + e));
                    // scale * P (dP - D) on pairs, in the scalar order (f32x2 rounds alike)
                    float dd[4];
                    const int j = ch * 32 + e;
                    uint64_t t01 = fsub2(f2pack(__uint_as_float(dpv[e]), __uint_as_float(dpv[e + 1])),
                                         f2pack(d4.x, d4.y));
                    uint64_t t23 = fsub2(f2pack(__uint_as_float(dpv[e + 2]), __uint_as_float(dpv[e + 3])),
                                         f2pack(d4.z, d4.w));
                    t01 = bwd_fmul2(bwd_fmul2(f2pack(pf[j], pf[j + 1]), t01), sc2);
                    t23 = bwd_fmul2(bwd_fmul2(f2pack(pf[j + 2], pf[j + 3]), t23), sc2);
                    f2unpack(t01, dd[0], dd[1]);
                    f2unpack(t23, dd[2], dd[3]);
                    dk[e / 2] = pack_bf16(dd[0], dd[1]);
                    dk[e / 2 + 1] = pack_bf16(dd[2], dd[3]);
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int unit = ch * 4 + u;
                    const uint32_t addr = atom + ((unit ^ (r & 7)) << 4);
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr),
                                 "r"(dk[4 * u]), "r"(dk[4 * u + 1]), "r"(dk[4 * u + 2]),
                                 "r"(dk[4 * u + 3]) : "memory");
                }
            }
            tc_fence_before();
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // dS visible to the MMA
            mbar_arrive(bar_p);

        }
        if (ok) {
            ok = mbar_wait_inl(bar_dkv, 0, abort_flag, wlim);
            ok = __all_sync(0xffffffffu, ok);
        }
        if (ok) {
            // warps 0-3 write dV_j, warps 4-7 dK_j (thread = K/V row r)
            tc_fence_after();
            const int kvrow = jb * BLOCK_M + r;
            const int64_t off = (static_cast<int64_t>(bh) * p.N + (kvrow < p.N ? kvrow : 0)) * D;
            __nv_bfloat16* out = (h ? p.dk : p.dv) + off;
            const uint32_t col = h ? C::DK_COL : C::DV_COL;
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

    tc_fence_before();
    __syncthreads();
    if (warp == BWD_MMA_WARP) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(TMEM_COLS) : "memory");
    }
}
