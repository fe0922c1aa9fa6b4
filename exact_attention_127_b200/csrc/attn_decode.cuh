/*
 * attn_decode.cuh -- split-K/V attention for decoding (one query row per head).
 * Included at the end of attn_fwd_sm100.cu, whose bounded mbarrier waits, TMA
 * wrappers, tensor-map encoder and device status word it uses.
 *
 * What is computed: for every head, one new query q attends to all N cached
 * keys and values, O = softmax(scale * q K^T) V and LSE = ln sum_j e^{s_j}
 * ("GPU 学习日报 Day 21", section 9 and FAQ Q5: decode is a matrix-vector
 * product bound by reading the K/V cache from device memory).  The key range is
 * cut into pieces that run in parallel and are merged afterwards ("Q31：
 * FlashAttention 为什么快", follow-up 3), with the merge rule of the online
 * softmax ("GPU 学习日报 Day 21", section 5.2): partial results that share a
 * reference max add, others are rescaled by 2^(m_old - m_new) first.
 *
 * The work is a stream over K and V with ~1 FLOP per byte, so it runs on the
 * CUDA cores and is bound by HBM; the tensor cores would add nothing.
 *
 *   decode_stream_kernel  persistent, one CTA per SM.  The K/V cache of all
 *                         heads is cut into stages of 32 keys per consumer warp
 *                         (128 keys and 4 warps at d = 128, 256 keys and 8 warps
 *                         at d = 64: 64 KB of K and V either way) and CTA c takes
 *                         the contiguous range [c P, (c+1) P) of the B*H*sph
 *                         stages (sph per head), so every SM streams the same
 *                         number of bytes.  The last warp loads each stage with
 *                         TMA into a 3-stage shared-memory ring; each consumer
 *                         warp takes 32 keys: lane i scores key i from its row
 *                         (the 128-byte swizzle spreads the 32 rows over all
 *                         banks and q is read as a broadcast), then the warp
 *                         walks the 32 keys, broadcasting p_i, while each lane
 *                         accumulates d/32 columns of p_i v_i.  At the end of
 *                         each head's part of the range the consumer warps
 *                         merge and write one unnormalised partial (O, m, l) to
 *                         slot head + c.
 *   decode_combine_kernel grid = B*H CTAs of d threads; merges the partials of
 *                         a head (CTAs c0 .. c1 of its stage range), divides by
 *                         l, rounds O to bf16 and writes LSE.
 *
 * The slot head + c is unique: the (head, CTA) pairs that share stages form a
 * staircase in which each step raises the head, the CTA or both, so their sums
 * are distinct and lie in [0, B*H + G - 1) for G CTAs.
 */

namespace {

constexpr int DEC_MAX_CTAS = 160;                       // >= the SMs of an sm_100 part; sizes the workspace
constexpr int DEC_BOX_ROWS = BLOCK_M;                   // rows of a box of the tensor maps encode_map makes
constexpr uint32_t DEC_BOX_BYTES = DEC_BOX_ROWS * 128;  // one box: 128 rows x 64 columns x 2 B

/* d = 128: 4 consumer warps, 128-key stages (two 64-column boxes per row);
 * d = 64: 8 consumer warps, 256-key stages (two 128-row boxes), so that a stage
 * is 64 KB either way and a warp's share of the per-key work stays the same. */
template <int D>
struct DecCfg {
    static constexpr int CONSUMERS = D == 64 ? 8 : 4;    // warps 0 .. CONSUMERS-1; the next one loads
    static constexpr int THREADS = (CONSUMERS + 1) * 32;
    static constexpr int STAGE_KEYS = 32 * CONSUMERS;    // one key per consumer lane
    static constexpr int ROW_BOXES = STAGE_KEYS / DEC_BOX_ROWS;
    static constexpr int COL_BOXES = D / 64;
    static constexpr uint32_t COL_BOX_STRIDE = STAGE_KEYS * 128;   // bytes between 64-column boxes
    static constexpr uint32_t KV_BYTES = COL_BOXES * COL_BOX_STRIDE;   // K (or V) of one stage
    static constexpr uint32_t STAGE_BYTES = 2 * KV_BYTES;
    static constexpr int NSTAGE = (192 * 1024) / STAGE_BYTES;    // 3
    static constexpr uint32_t Q_OFF = NSTAGE * STAGE_BYTES;      // q * scale * log2(e), fp32
    static constexpr uint32_t RED_OFF = Q_OFF + D * 4;           // per warp: O row, then m, l
    static constexpr uint32_t RED_BYTES = CONSUMERS * (D + 2) * 4;
    static constexpr uint32_t BAR_OFF = (RED_OFF + RED_BYTES + 7u) & ~7u;
    static constexpr uint32_t FLAG_OFF = BAR_OFF + 16 * NSTAGE;  // full[NSTAGE], empty[NSTAGE]
    static constexpr int SMEM_BYTES = FLAG_OFF + 16 + 1024;      // + slack for the 1 KB alignment
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
};

__device__ __forceinline__ float dec_ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

/* Named barrier over the consumer warps (the loader never joins it). */
template <int THREADS>
__device__ __forceinline__ void dec_consumers_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(THREADS) : "memory");
}

template <int D>
__global__ void __launch_bounds__(DecCfg<D>::THREADS, 1)
decode_stream_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                     const __nv_bfloat16* __restrict__ q, float* __restrict__ part_o,
                     float2* __restrict__ part_ml, int N, int sph, int per_cta, int total,
                     float scale_log2, uint64_t wlim, int withhold) {
    using C = DecCfg<D>;
    constexpr int CPL = D / 32;                  // output columns per lane
    constexpr int NCW = C::CONSUMERS;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;        // the swizzle wants 1 KB alignment
    uint8_t* const bp = smem_raw + (base - raw);
    const uint32_t bars = base + C::BAR_OFF;
    auto bar_full = [&](int s) { return bars + 8u * s; };
    auto bar_empty = [&](int s) { return bars + 8u * (C::NSTAGE + s); };
    volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(bp + C::FLAG_OFF);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int lo = blockIdx.x * per_cta;
    const int hi = lo + min(per_cta, total - lo);        // lo < total for every CTA launched

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::NSTAGE; ++s) {
            mbar_init(bar_full(s), 1);
            mbar_init(bar_empty(s), NCW);                // lane 0 of each consumer warp
        }
        *abort_flag = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    __syncthreads();

    if (warp == NCW) {
        /* ---------------- loader: stage g = (head g / sph, keys 128 (g % sph) ..) ---------------- */
        if (lane == 0) {
            prefetch_tmap(&tm_k);
            prefetch_tmap(&tm_v);
            int it = 0;
            const int hi_load = withhold ? lo : hi;      // test hook: load nothing, so waits run out
            for (int g = lo; g < hi_load; ++g, ++it) {
                const int s = it % C::NSTAGE;
                if (it >= C::NSTAGE &&
                    !mbar_wait(bar_empty(s), ((it / C::NSTAGE) - 1) & 1, abort_flag, wlim))
                    break;
                const int bh = g / sph, key0 = (g - bh * sph) * C::STAGE_KEYS;
                const uint32_t dst = base + s * C::STAGE_BYTES;
                mbar_arrive_expect_tx(bar_full(s), C::STAGE_BYTES);
#pragma unroll
                for (int b = 0; b < C::COL_BOXES; ++b)
#pragma unroll
                    for (int rb = 0; rb < C::ROW_BOXES; ++rb) {
                        const uint32_t off = b * C::COL_BOX_STRIDE + rb * DEC_BOX_BYTES;
                        tma_load_3d(&tm_k, dst + off, bar_full(s), 64 * b, key0 + rb * DEC_BOX_ROWS, bh);
                        tma_load_3d(&tm_v, dst + C::KV_BYTES + off, bar_full(s), 64 * b,
                                    key0 + rb * DEC_BOX_ROWS, bh);
                    }
            }
            // the copies in flight land before the CTA may exit (after an abort too)
            for (int j = max(0, it - C::NSTAGE); j < it; ++j)
                mbar_drain_wait(bar_full(j % C::NSTAGE), (j / C::NSTAGE) & 1, wlim);
        }
        return;
    }

    /* ---------------- consumer warps: 32 keys of every stage each ---------------- */
    float* const q_s = reinterpret_cast<float*>(bp + C::Q_OFF);
    float* const red_o = reinterpret_cast<float*>(bp + C::RED_OFF);      // [NCW][D]
    float* const red_m = red_o + NCW * D;                                // [NCW]
    float* const red_l = red_m + NCW;                                    // [NCW]
    const int r = 32 * warp + lane;              // this lane's key row within a stage
    bool ok = true;
    float m_w = -INFINITY;                       // warp-uniform reference max (log2 units)
    float l_lane = 0.0f;                         // this lane's share of the row sum
    float acc[CPL];
#pragma unroll
    for (int e = 0; e < CPL; ++e) acc[e] = 0.0f;
    int it = 0;
    for (int g = lo; g < hi; ++g, ++it) {
        const int bh = g / sph, sidx = g - bh * sph;
        if (g == lo || sidx == 0) {
            // a new head: the previous one is merged and done with q_s
            dec_consumers_sync<NCW * 32>();
            for (int c = threadIdx.x; c < D; c += NCW * 32)
                q_s[c] = __bfloat162float(q[static_cast<int64_t>(bh) * D + c]) * scale_log2;
            dec_consumers_sync<NCW * 32>();
            m_w = -INFINITY;
            l_lane = 0.0f;
#pragma unroll
            for (int e = 0; e < CPL; ++e) acc[e] = 0.0f;
        }
        const int s = it % C::NSTAGE;
        if (ok) ok = mbar_wait(bar_full(s), (it / C::NSTAGE) & 1, abort_flag, wlim);
        ok = __all_sync(0xffffffffu, ok);
        const int nvalid = min(32, N - (sidx * C::STAGE_KEYS + 32 * warp));   // keys of this warp
        if (ok && nvalid > 0) {
            const uint8_t* kst = bp + s * C::STAGE_BYTES;
            const uint8_t* vst = kst + C::KV_BYTES;
            // score of key r: its row, 16 bytes at a time; 16-byte unit u of a 128-byte
            // row sits at position u ^ (r % 8) (rows past N are zeros from the TMA)
            float a[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
            for (int u = 0; u < D / 8; ++u) {
                const uint4 w = *reinterpret_cast<const uint4*>(
                    kst + (u >> 3) * C::COL_BOX_STRIDE + r * 128 + (((u & 7) ^ (r & 7)) << 4));
                const float4 qa = *reinterpret_cast<const float4*>(q_s + 8 * u);
                const float4 qb = *reinterpret_cast<const float4*>(q_s + 8 * u + 4);
                a[0] = fmaf(bf16_lo(w.x), qa.x, a[0]);
                a[1] = fmaf(bf16_hi(w.x), qa.y, a[1]);
                a[2] = fmaf(bf16_lo(w.y), qa.z, a[2]);
                a[3] = fmaf(bf16_hi(w.y), qa.w, a[3]);
                a[0] = fmaf(bf16_lo(w.z), qb.x, a[0]);
                a[1] = fmaf(bf16_hi(w.z), qb.y, a[1]);
                a[2] = fmaf(bf16_lo(w.w), qb.z, a[2]);
                a[3] = fmaf(bf16_hi(w.w), qb.w, a[3]);
            }
            const float sc = lane < nvalid ? (a[0] + a[1]) + (a[2] + a[3]) : -INFINITY;
            // online update with the max of the 32 keys (lane 0's key is valid)
            float mt = sc;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, off));
            const float m_new = fmaxf(m_w, mt);
            const float alpha = dec_ex2(m_w - m_new);            // 0 on the first keys of a head
            const float p = lane < nvalid ? dec_ex2(sc - m_new) : 0.0f;
            l_lane = l_lane * alpha + p;
#pragma unroll
            for (int e = 0; e < CPL; ++e) acc[e] *= alpha;
            m_w = m_new;
            // O += p_i v_i; lane owns columns [CPL lane, CPL lane + CPL).  Rows past N
            // are zeros and carry p = 0.
#pragma unroll 8
            for (int i = 0; i < 32; ++i) {
                const float pi = __shfl_sync(0xffffffffu, p, i);
                const int rv = 32 * warp + i;
                if (CPL == 4) {
                    const uint2 w = *reinterpret_cast<const uint2*>(
                        vst + (lane >> 4) * C::COL_BOX_STRIDE + rv * 128 +
                        ((((lane & 15) >> 1) ^ (rv & 7)) << 4) + (lane & 1) * 8);
                    acc[0] = fmaf(pi, bf16_lo(w.x), acc[0]);
                    acc[1] = fmaf(pi, bf16_hi(w.x), acc[1]);
                    acc[2] = fmaf(pi, bf16_lo(w.y), acc[2]);
                    acc[3] = fmaf(pi, bf16_hi(w.y), acc[3]);
                } else {
                    const uint32_t w = *reinterpret_cast<const uint32_t*>(
                        vst + rv * 128 + (((lane >> 2) ^ (rv & 7)) << 4) + (lane & 3) * 4);
                    acc[0] = fmaf(pi, bf16_lo(w), acc[0]);
                    acc[1] = fmaf(pi, bf16_hi(w), acc[1]);
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_empty(s));            // the stage may be reloaded
        if (g + 1 == hi || sidx + 1 == sph) {
            // the end of this head's part of the range: one partial from the four warps
            float l_w = l_lane;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) l_w += __shfl_xor_sync(0xffffffffu, l_w, off);
#pragma unroll
            for (int e = 0; e < CPL; ++e) red_o[warp * D + CPL * lane + e] = acc[e];
            if (lane == 0) {
                red_m[warp] = m_w;
                red_l[warp] = l_w;
            }
            dec_consumers_sync<NCW * 32>();
            float M = -INFINITY;
#pragma unroll
            for (int w = 0; w < NCW; ++w) M = fmaxf(M, red_m[w]);
            const int64_t slot = static_cast<int64_t>(bh) + blockIdx.x;
            for (int c = threadIdx.x; c < D; c += NCW * 32) {
                float o = 0.0f;
#pragma unroll
                for (int w = 0; w < NCW; ++w)
                    if (red_m[w] != -INFINITY) o += red_o[w * D + c] * dec_ex2(red_m[w] - M);
                part_o[slot * D + c] = o;
            }
            if (threadIdx.x == 0) {
                float Lsum = 0.0f;
#pragma unroll
                for (int w = 0; w < NCW; ++w)
                    if (red_m[w] != -INFINITY) Lsum += red_l[w] * dec_ex2(red_m[w] - M);
                part_ml[slot] = make_float2(M, Lsum);
            }
        }
    }
}

/* Merge the partials of head bh: CTAs c0 .. c1 cover its stages
 * [bh sph, (bh + 1) sph), and CTA c wrote slot bh + c. */
template <int D>
__global__ void __launch_bounds__(D)
decode_combine_kernel(const float* __restrict__ part_o, const float2* __restrict__ part_ml,
                      __nv_bfloat16* __restrict__ o, float* __restrict__ lse, int sph, int per_cta) {
    const int64_t bh = blockIdx.x;
    const int c = threadIdx.x;
    const int c0 = static_cast<int>(bh * sph / per_cta);
    const int c1 = static_cast<int>(((bh + 1) * sph - 1) / per_cta);
    float M = -INFINITY;
    for (int cta = c0; cta <= c1; ++cta) M = fmaxf(M, part_ml[bh + cta].x);
    float Lsum = 0.0f, acc = 0.0f;
    for (int cta = c0; cta <= c1; ++cta) {
        const float2 v = part_ml[bh + cta];
        if (v.x == -INFINITY) continue;
        const float w = dec_ex2(v.x - M);
        Lsum += v.y * w;
        acc += part_o[(bh + cta) * D + c] * w;
    }
    o[bh * D + c] = __float2bfloat16_rn(Lsum > 0.0f ? acc / Lsum : 0.0f);
    if (c == 0) lse[bh] = (M + log2f(Lsum)) * LN2;
}

/* Work plan: stages per head, stages per CTA and the number of CTAs. */
struct DecodePlan {
    int sph;       // ceil(N / 128)
    int total;     // B*H*sph
    int per_cta;   // P
    int ctas;      // G = ceil(total / P) <= min(SMs, DEC_MAX_CTAS)
};

DecodePlan decode_plan(int64_t BH, int64_t N, int stage_keys, int num_sms) {
    DecodePlan pl;
    pl.sph = static_cast<int>((N + stage_keys - 1) / stage_keys);
    pl.total = static_cast<int>(BH * pl.sph);
    int64_t g0 = std::min<int64_t>(std::min(num_sms, DEC_MAX_CTAS), pl.total);
    if (g0 < 1) g0 = 1;
    pl.per_cta = static_cast<int>((pl.total + g0 - 1) / g0);
    pl.ctas = (pl.total + pl.per_cta - 1) / pl.per_cta;
    return pl;
}

int decode_validate(int64_t B, int64_t H, int64_t N, int64_t d, float scale, bool* empty) {
    if (B < 0 || H < 0 || N < 0) return ATTN_ERR_SHAPE;
    if (d != 64 && d != 128) return ATTN_ERR_HEADDIM;
    if (!(scale > 0.0f) || !isfinite(scale)) return ATTN_ERR_SCALE;
    *empty = (B == 0 || H == 0 || N == 0);
    if (*empty) return ATTN_OK;
    if (N > INT32_MAX / 2 || H > INT32_MAX / B) return ATTN_ERR_SHAPE;
    const int64_t BH = B * H;
    const int64_t sph = (N + DEC_BOX_ROWS - 1) / DEC_BOX_ROWS;          // the most stages a head can have
    if (BH > (INT32_MAX - DEC_MAX_CTAS) / sph) return ATTN_ERR_SHAPE;   // stage and slot indices fit int32
    return ATTN_OK;
}

/* Partials: B*H + DEC_MAX_CTAS - 1 slots of d fp32 values, then as many (m, l). */
size_t decode_ws_bytes(int64_t BH, int64_t d) {
    const size_t slots = static_cast<size_t>(BH) + DEC_MAX_CTAS - 1;
    const size_t po = slots * d * sizeof(float);
    return ((po + 255u) & ~static_cast<size_t>(255u)) + slots * sizeof(float2);
}

template <int D>
int decode_launch(const CUtensorMap& mk, const CUtensorMap& mv, const __nv_bfloat16* q,
                  float* part_o, float2* part_ml, __nv_bfloat16* o, float* lse, int64_t BH,
                  int N, const DecodePlan& pl, float scale_log2, DeviceInfo* di, cudaStream_t s,
                  uint64_t wait_limit_ns, int withhold) {
    auto kern = decode_stream_kernel<D>;
    constexpr int SMEM = DecCfg<D>::SMEM_BYTES;
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        bool& set = di->dec_set[D == 128 ? 1 : 0];
        if (!set) {
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM) !=
                cudaSuccess) {
                cudaGetLastError();
                return ATTN_ERR_LAUNCH;
            }
            set = true;
        }
    }
    kern<<<pl.ctas, DecCfg<D>::THREADS, SMEM, s>>>(mk, mv, q, part_o, part_ml, N, pl.sph, pl.per_cta,
                                            pl.total, scale_log2, wait_limit_ns, withhold);
    decode_combine_kernel<D><<<static_cast<unsigned>(BH), D, 0, s>>>(part_o, part_ml, o, lse, pl.sph,
                                                                    pl.per_cta);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_LAUNCH;
    return ATTN_OK;
}

/* The decode call behind attn_decode and its timeout test hook. */
int decode_impl(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B,
                int64_t H, int64_t N, int64_t d, float scale, void* workspace,
                size_t workspace_bytes, void* stream, uint64_t wait_limit_ns, int withhold) {
    bool empty = false;
    int st = decode_validate(B, H, N, d, scale, &empty);
    if (st != ATTN_OK || empty) return st;
    if (!q || !k || !v || !o || !lse) return ATTN_ERR_NULL;
    const void* ptrs[5] = {q, k, v, o, lse};
    for (const void* ptr : ptrs)
        if (reinterpret_cast<uintptr_t>(ptr) & 15u) return ATTN_ERR_ALIGN;
    const int64_t BH = B * H;
    const size_t ws_need = decode_ws_bytes(BH, d);
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < ws_need)
        return ATTN_ERR_WORKSPACE;
    {
        // outputs (o, lse, the workspace) may not overlap the inputs or each other
        const void* outs[3] = {o, lse, workspace};
        const size_t out_bytes[3] = {static_cast<size_t>(BH * d) * 2, static_cast<size_t>(BH) * 4,
                                     ws_need};
        const void* ins[3] = {q, k, v};
        const size_t in_bytes[3] = {static_cast<size_t>(BH * d) * 2,
                                    static_cast<size_t>(BH * N * d) * 2,
                                    static_cast<size_t>(BH * N * d) * 2};
        if ((st = check_overlaps(outs, out_bytes, 3, ins, in_bytes, 3)) != ATTN_OK) return st;
    }
    int dev = 0;
    DeviceInfo* di = nullptr;
    if ((st = device_info(&dev, &di)) != ATTN_OK) return st;
    EncodeTiledFn enc = nullptr;
    if ((st = get_encode(&enc)) != ATTN_OK) return st;
    CUtensorMap mk, mv;
    if ((st = encode_map(enc, &mk, k, BH, N, d)) != ATTN_OK) return st;
    if ((st = encode_map(enc, &mv, v, BH, N, d)) != ATTN_OK) return st;

    const DecodePlan pl = decode_plan(BH, N, d == 64 ? DecCfg<64>::STAGE_KEYS : DecCfg<128>::STAGE_KEYS,
                                      di->num_sms);
    const size_t slots = static_cast<size_t>(BH) + DEC_MAX_CTAS - 1;
    float* part_o = static_cast<float*>(workspace);
    float2* part_ml = reinterpret_cast<float2*>(
        static_cast<char*>(workspace) + ((slots * d * sizeof(float) + 255u) & ~static_cast<size_t>(255u)));
    const float sl = scale * LOG2E;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const auto* qb = static_cast<const __nv_bfloat16*>(q);
    auto* ob = static_cast<__nv_bfloat16*>(o);
    return d == 64 ? decode_launch<64>(mk, mv, qb, part_o, part_ml, ob, lse, BH, static_cast<int>(N), pl,
                                       sl, di, s, wait_limit_ns, withhold)
                   : decode_launch<128>(mk, mv, qb, part_o, part_ml, ob, lse, BH, static_cast<int>(N), pl,
                                        sl, di, s, wait_limit_ns, withhold);
}

}  // namespace

extern "C" {

size_t attn_decode_workspace_bytes(int64_t B, int64_t H, int64_t N, int64_t d) {
    bool empty = false;
    if (decode_validate(B, H, N, d, 1.0f, &empty) != ATTN_OK) return 0;
    if (empty) return 0;
    return decode_ws_bytes(B * H, d);
}

int attn_decode(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B,
                int64_t H, int64_t N, int64_t d, float scale, void* workspace,
                size_t workspace_bytes, void* stream) {
    return decode_impl(q, k, v, o, lse, B, H, N, d, scale, workspace, workspace_bytes, stream,
                       WAIT_LIMIT_NS, 0);
}

int attn_decode_test_wait_timeout(const void* q, const void* k, const void* v, void* o, float* lse,
                                  int64_t B, int64_t H, int64_t N, int64_t d, void* workspace,
                                  size_t workspace_bytes, void* stream) {
    return decode_impl(q, k, v, o, lse, B, H, N, d, 0.125f, workspace, workspace_bytes, stream,
                       TEST_WAIT_LIMIT_NS, 1);
}

}  // extern "C"

/*
 * Allocation-free decode.  Some callers cannot allocate device memory
 * themselves: a plugin or runtime whose host application owns all device
 * memory through its own pool, or a latency-bound loop that must not call
 * cudaMalloc (which can synchronise the device) once it is running.  For them
 * the partial results live in this fixed buffer, part of the library's own
 * device image.  It is created with the module on every GPU that loads the
 * library and stays until the process exits.
 */
constexpr size_t DECODE_STATIC_SCRATCH_BYTES = size_t(8) << 20;   // 8 MiB
static __device__ __align__(256) unsigned char g_decode_scratch[DECODE_STATIC_SCRATCH_BYTES];

namespace {
/* Device address of g_decode_scratch in the context current on this thread.
 * In host code the array's name only stands in for the symbol (it is not a
 * device address), so the address is looked up with cudaGetSymbolAddress once
 * per device and context, with that device current, and cached; a context
 * reset or another current context leads to a fresh lookup (device_info). */
int scratch_address(void** out) {
    int dev = 0;
    DeviceInfo* di = nullptr;
    const int st = device_info(&dev, &di);
    if (st != ATTN_OK) return st;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!di->scratch) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_decode_scratch) != cudaSuccess || !ptr) {
            cudaGetLastError();
            return ATTN_ERR_CUDA;
        }
        di->scratch = ptr;
    }
    *out = di->scratch;
    return ATTN_OK;
}
}  // namespace

extern "C" {

size_t attn_decode_noalloc_scratch_bytes(void) { return DECODE_STATIC_SCRATCH_BYTES; }

int attn_decode_noalloc(const void* q, const void* k, const void* v, void* o, float* lse,
                        int64_t B, int64_t H, int64_t N, int64_t d, float scale, void* stream) {
    bool empty = false;
    int st = decode_validate(B, H, N, d, scale, &empty);
    if (st != ATTN_OK || empty) return st;
    if (decode_ws_bytes(B * H, d) > DECODE_STATIC_SCRATCH_BYTES) return ATTN_ERR_WORKSPACE;
    void* scratch = nullptr;
    if ((st = scratch_address(&scratch)) != ATTN_OK) return st;
    return attn_decode(q, k, v, o, lse, B, H, N, d, scale, scratch, DECODE_STATIC_SCRATCH_BYTES,
                       stream);
}

}  // extern "C"
