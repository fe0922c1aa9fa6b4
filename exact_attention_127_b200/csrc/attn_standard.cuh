/*
 * attn_standard.cuh -- the unfused "standard attention" path, for comparison.
 *
 * "GPU 学习日报 Day 21", sections 3.1 and 4.2, describe the standard
 * implementation as three kernels whose N x N intermediates round-trip through
 * device memory:
 *   kernel 1: S = Q K^T * scale        -> HBM
 *   kernel 2: P = softmax(S) (rows)    HBM -> HBM
 *   kernel 3: O = P V                  HBM -> HBM
 * This file builds exactly that, hand-written for sm_100a (tcgen05 GEMMs fed by
 * TMA, a row-softmax kernel), so that the fused kernel can be measured against
 * it on the same GPU.  S is kept in fp32 (not the 16-bit matrix the page's
 * memory estimate assumes) so that this path meets the same accuracy bar as
 * the fused one; P overwrites the first half of each S row in place as bf16.
 * Causal rows mask keys j > i in kernel 2 only: kernels 1 and 3 compute the
 * full N x N products, as the standard path does.
 *
 * Included into attn_fwd_sm100.cu (same translation unit) to share the mbarrier,
 * TMA and tcgen05 helpers and the device status word.
 */

constexpr int STD_THREADS = 192;      // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue
constexpr int STD_PV_STAGES = 4;
constexpr int STD_PV_KEYS = 64;       // keys per K step of O = P V (one 128B swizzle atom of P)
constexpr int STD_SOFTMAX_THREADS = 256;
constexpr int STD_MAX_N = 32768;

struct StdParams {
    float* S;              // [BH, Np, Np] fp32; P (bf16) overwrites each row's first half
    float* lse;            // [BH, N]
    __nv_bfloat16* o;      // [BH, N, D]
    int N, Np, BH;
    int causal;
    float scale;
    uint64_t wait_limit_ns;
};

/* Kernel 1: one 128 x 128 tile of S = scale * Q K^T per CTA, written in fp32. */
template <int D>
__global__ void __launch_bounds__(STD_THREADS, 1)
std_qk_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const StdParams p) {
    constexpr uint32_t TILE = BLOCK_M * D * 2;
    constexpr int CHUNKS = D / CHUNK_ELEMS;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* const base_ptr = smem_raw + (base - raw);
    const uint32_t sQ = base, sK = base + TILE;
    const uint32_t bar_full = base + 2 * TILE, bar_done = bar_full + 8, bar_drain = bar_full + 16;
    uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + 2 * TILE + 32);
    volatile uint32_t* const abort_flag = reinterpret_cast<volatile uint32_t*>(base_ptr + 2 * TILE + 36);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint64_t wlim = p.wait_limit_ns;
    const int jt = blockIdx.x, it = blockIdx.y, bh = blockIdx.z;

    if (threadIdx.x == 0) {
        mbar_init(bar_full, 1);
        mbar_init(bar_done, 1);
        mbar_init(bar_drain, 1);
        *abort_flag = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(tmem_slot)), "r"(128) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            mbar_arrive_expect_tx(bar_full, 2 * TILE);
            for (int c = 0; c < CHUNKS; ++c) {
                tma_load_3d(&tm_q, sQ + c * CHUNK_BYTES, bar_full, c * CHUNK_ELEMS, it * BLOCK_M, bh);
                tma_load_3d(&tm_k, sK + c * CHUNK_BYTES, bar_full, c * CHUNK_ELEMS, jt * BLOCK_N, bh);
            }
            // the copies must land before the CTA exits, whatever happens elsewhere
            mbar_drain_wait(bar_full, 0, wlim);
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            if (mbar_wait(bar_full, 0, abort_flag, wlim)) {
                issue_qk<D>(tmem, sdesc_sw128(sQ, 16, 1024), sdesc_sw128(sK, 16, 1024),
                            idesc_bf16(BLOCK_M, BLOCK_N, false));
                mma_commit(bar_done);
            }
            mma_commit(bar_drain);
            mbar_drain_wait(bar_drain, 0, wlim);
        }
        __syncwarp();
    } else {
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        bool ok = mbar_wait(bar_done, 0, abort_flag, wlim);
        ok = __all_sync(0xffffffffu, ok);
        if (ok) {
            tc_fence_after();
            const int row = it * BLOCK_M + r;
            float* dst = p.S + (static_cast<size_t>(bh) * p.Np + row) * p.Np + jt * BLOCK_N;
            const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
#pragma unroll
            for (int ch = 0; ch < BLOCK_N / 32; ++ch) {
                uint32_t v[32];
                tmem_ld32_wait(taddr + ch * 32, v);
                float4* d4 = reinterpret_cast<float4*>(dst + ch * 32);
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    d4[e] = make_float4(__uint_as_float(v[4 * e]) * p.scale,
                                        __uint_as_float(v[4 * e + 1]) * p.scale,
                                        __uint_as_float(v[4 * e + 2]) * p.scale,
                                        __uint_as_float(v[4 * e + 3]) * p.scale);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(128)
                     : "memory");
    }
}

/* Kernel 2: one row per CTA -- row max, exponentials, row sum, P = e^{s-m}/l
 * written as bf16 over the row's first half, and LSE = m + ln l.  VEC float4
 * per thread covers rows of up to 1024 VEC scores; the smallest VEC that
 * covers the row keeps registers, and so resident rows per SM, high.  Masked
 * scores (causal, j > i) are not read: their P is written as 0. */
template <int VEC>
__global__ void __launch_bounds__(STD_SOFTMAX_THREADS)
std_softmax_kernel(const StdParams p) {
    __shared__ float red[STD_SOFTMAX_THREADS / 32];
    const int64_t row = blockIdx.x;
    const int bh = static_cast<int>(row / p.N), i = static_cast<int>(row % p.N);
    float* srow = p.S + (static_cast<size_t>(bh) * p.Np + i) * p.Np;
    const int n_valid = p.causal ? i + 1 : p.N;
    const int nvec = p.Np / 4;
    float4 x[VEC];
    float m = -INFINITY;
#pragma unroll
    for (int u = 0; u < VEC; ++u) {
        const int g = threadIdx.x + STD_SOFTMAX_THREADS * u;
        float4 t = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
        if (g < nvec && 4 * g < n_valid) {
            t = reinterpret_cast<const float4*>(srow)[g];
            const int e = 4 * g;
            if (e >= n_valid) t.x = -INFINITY;
            if (e + 1 >= n_valid) t.y = -INFINITY;
            if (e + 2 >= n_valid) t.z = -INFINITY;
            if (e + 3 >= n_valid) t.w = -INFINITY;
        }
        x[u] = t;
        m = fmaxf(m, fmaxf(fmaxf(t.x, t.y), fmaxf(t.z, t.w)));
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    if (lane == 0) red[warp] = m;
    __syncthreads();                       // also: every thread has read its S values
    m = red[0];
#pragma unroll
    for (int w = 1; w < STD_SOFTMAX_THREADS / 32; ++w) m = fmaxf(m, red[w]);
    __syncthreads();
    const float mb = m * LOG2E;
    float l = 0.0f;
#pragma unroll
    for (int u = 0; u < VEC; ++u) {
        float4& t = x[u];
        t.x = ex2(fmaf(t.x, LOG2E, -mb));
        t.y = ex2(fmaf(t.y, LOG2E, -mb));
        t.z = ex2(fmaf(t.z, LOG2E, -mb));
        t.w = ex2(fmaf(t.w, LOG2E, -mb));
        l += (t.x + t.y) + (t.z + t.w);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
    if (lane == 0) red[warp] = l;
    __syncthreads();
    l = 0.0f;
#pragma unroll
    for (int w = 0; w < STD_SOFTMAX_THREADS / 32; ++w) l += red[w];
    const float inv = 1.0f / l;
    uint2* prow = reinterpret_cast<uint2*>(srow);   // bf16 P over the row's first half
#pragma unroll
    for (int u = 0; u < VEC; ++u) {
        const int g = threadIdx.x + STD_SOFTMAX_THREADS * u;
        if (g < nvec)
            prow[g] = make_uint2(pack_bf16(x[u].x * inv, x[u].y * inv),
                                 pack_bf16(x[u].z * inv, x[u].w * inv));
    }
    if (threadIdx.x == 0) p.lse[row] = m + logf(l);
}

/* Kernel 2 for short rows (Np <= 2048): one warp per row, eight rows per CTA;
 * the same arithmetic as std_softmax_kernel with warp-level reductions. */
constexpr int STD_SHORT_MAX_NP = 2048;
__global__ void __launch_bounds__(STD_SOFTMAX_THREADS)
std_softmax_short_kernel(const StdParams p) {
    constexpr int VEC = STD_SHORT_MAX_NP / (4 * 32);   // float4 per lane, max
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * (STD_SOFTMAX_THREADS / 32) + warp;
    if (row >= static_cast<int64_t>(p.BH) * p.N) return;
    const int bh = static_cast<int>(row / p.N), i = static_cast<int>(row % p.N);
    float* srow = p.S + (static_cast<size_t>(bh) * p.Np + i) * p.Np;
    const int n_valid = p.causal ? i + 1 : p.N;
    const int nvec = p.Np / 4;
    float4 x[VEC];
    float m = -INFINITY;
#pragma unroll
    for (int u = 0; u < VEC; ++u) {
        const int g = lane + 32 * u;
        float4 t = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
        if (g < nvec) {
            t = reinterpret_cast<const float4*>(srow)[g];
            const int e = 4 * g;
            if (e >= n_valid) t.x = -INFINITY;
            if (e + 1 >= n_valid) t.y = -INFINITY;
            if (e + 2 >= n_valid) t.z = -INFINITY;
            if (e + 3 >= n_valid) t.w = -INFINITY;
        }
        x[u] = t;
        m = fmaxf(m, fmaxf(fmaxf(t.x, t.y), fmaxf(t.z, t.w)));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    const float mb = m * LOG2E;
    float l = 0.0f;
#pragma unroll
    for (int u = 0; u < VEC; ++u) {
        float4& t = x[u];
        t.x = ex2(fmaf(t.x, LOG2E, -mb));
        t.y = ex2(fmaf(t.y, LOG2E, -mb));
        t.z = ex2(fmaf(t.z, LOG2E, -mb));
        t.w = ex2(fmaf(t.w, LOG2E, -mb));
        l += (t.x + t.y) + (t.z + t.w);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
    const float inv = 1.0f / l;
    __syncwarp();                          // the whole row is read before P overwrites it
    uint2* prow = reinterpret_cast<uint2*>(srow);
#pragma unroll
    for (int u = 0; u < VEC; ++u) {
        const int g = lane + 32 * u;
        if (g < nvec)
            prow[g] = make_uint2(pack_bf16(x[u].x * inv, x[u].y * inv),
                                 pack_bf16(x[u].z * inv, x[u].w * inv));
    }
    if (lane == 0) p.lse[row] = m + logf(l);
}

/* Kernel 3: one 128-row tile of O = P V per CTA, K steps of 64 keys through a
 * TMA ring; P (bf16, K-major) and V (bf16, MN-major) from shared memory. */
template <int D>
__global__ void __launch_bounds__(STD_THREADS, 1)
std_pv_kernel(const __grid_constant__ CUtensorMap tm_p, const __grid_constant__ CUtensorMap tm_v,
              const StdParams p) {
    constexpr uint32_t A_BYTES = BLOCK_M * STD_PV_KEYS * 2;       // 16 KB
    constexpr uint32_t B_BYTES = STD_PV_KEYS * D * 2;             // 8 or 16 KB
    constexpr uint32_t STAGE = A_BYTES + B_BYTES;
    constexpr uint32_t B_CHUNK = STD_PV_KEYS * 128;               // one 64-column box of V
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* const base_ptr = smem_raw + (base - raw);
    const uint32_t bars = base + STD_PV_STAGES * STAGE;
    auto bar_full = [&](int s) { return bars + 8u * s; };
    auto bar_empty = [&](int s) { return bars + 8u * (STD_PV_STAGES + s); };
    const uint32_t bar_done = bars + 16 * STD_PV_STAGES, bar_drain = bar_done + 8;
    uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + STD_PV_STAGES * STAGE + 16 * STD_PV_STAGES + 32);
    volatile uint32_t* const abort_flag = reinterpret_cast<volatile uint32_t*>(tmem_slot + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint64_t wlim = p.wait_limit_ns;
    const int it = blockIdx.x, bh = blockIdx.y;
    const int nk = p.Np / STD_PV_KEYS;
    constexpr uint32_t TMEM_COLS_PV = D;   // 64 or 128: a power of two >= 32

    if (threadIdx.x == 0) {
        for (int s = 0; s < STD_PV_STAGES; ++s) {
            mbar_init(bar_full(s), 1);
            mbar_init(bar_empty(s), 1);
        }
        mbar_init(bar_done, 1);
        mbar_init(bar_drain, 1);
        *abort_flag = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(tmem_slot)), "r"(TMEM_COLS_PV) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            int issued = 0;
            for (int kc = 0; kc < nk; ++kc) {
                const int s = kc % STD_PV_STAGES;
                if (!mbar_wait(bar_empty(s), ((kc / STD_PV_STAGES) & 1) ^ 1, abort_flag, wlim)) break;
                const uint32_t a = base + s * STAGE, b = a + A_BYTES;
                mbar_arrive_expect_tx(bar_full(s), STAGE);
                tma_load_3d(&tm_p, a, bar_full(s), kc * STD_PV_KEYS, it * BLOCK_M, bh);
                for (int c = 0; c < D / CHUNK_ELEMS; ++c)
                    tma_load_3d(&tm_v, b + c * B_CHUNK, bar_full(s), c * CHUNK_ELEMS,
                                kc * STD_PV_KEYS, bh);
                ++issued;
            }
            // let every copy this thread issued land before the CTA can exit
            const int back = issued < STD_PV_STAGES ? issued : STD_PV_STAGES;
            for (int b = 1; b <= back; ++b) {
                const int kc = issued - b;
                mbar_drain_wait(bar_full(kc % STD_PV_STAGES), (kc / STD_PV_STAGES) & 1, wlim);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(BLOCK_M, D, true);
            bool ok = true;
            for (int kc = 0; kc < nk && ok; ++kc) {
                const int s = kc % STD_PV_STAGES;
                ok = mbar_wait(bar_full(s), (kc / STD_PV_STAGES) & 1, abort_flag, wlim);
                if (!ok) break;
                const uint32_t a = base + s * STAGE, b = a + A_BYTES;
                const uint64_t ad = sdesc_sw128(a, 16, 1024);
                const uint64_t bd = sdesc_sw128(b, B_CHUNK, 1024);
#pragma unroll
                for (int kk = 0; kk < STD_PV_KEYS / 16; ++kk)
                    mma_ss(tmem, ad + ((kk * 32) >> 4), bd + ((kk * 16 * 128) >> 4), idesc,
                           (kc > 0 || kk > 0) ? 1u : 0u);
                mma_commit(bar_empty(s));
            }
            if (ok) mma_commit(bar_done);
            mma_commit(bar_drain);
            mbar_drain_wait(bar_drain, 0, wlim);
        }
        __syncwarp();
    } else {
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        bool ok = mbar_wait(bar_done, 0, abort_flag, wlim);
        ok = __all_sync(0xffffffffu, ok);
        if (ok) {
            tc_fence_after();
            const int row = it * BLOCK_M + r;
            const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
            __nv_bfloat16* orow = p.o + (static_cast<size_t>(bh) * p.N + (row < p.N ? row : 0)) * D;
#pragma unroll
            for (int ch = 0; ch < D / 32; ++ch) {
                uint32_t v[32];
                tmem_ld32_wait(taddr + ch * 32, v);
                if (row < p.N) {
                    uint4* dst = reinterpret_cast<uint4*>(orow + ch * 32);
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        dst[e] = make_uint4(
                            pack_bf16(__uint_as_float(v[8 * e + 0]), __uint_as_float(v[8 * e + 1])),
                            pack_bf16(__uint_as_float(v[8 * e + 2]), __uint_as_float(v[8 * e + 3])),
                            pack_bf16(__uint_as_float(v[8 * e + 4]), __uint_as_float(v[8 * e + 5])),
                            pack_bf16(__uint_as_float(v[8 * e + 6]), __uint_as_float(v[8 * e + 7])));
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(TMEM_COLS_PV) : "memory");
    }
}
