/*
 * attn_decode.cu -- split-K/V attention for decoding (one query row per head).
 *
 * What is computed: for every head, one new query q attends to all N cached
 * keys and values, O = softmax(scale * q K^T) V and LSE = ln sum_j e^{s_j}
 * ("GPU 学习日报 Day 21", section 9 and FAQ Q5: decode is a matrix-vector
 * product bound by reading the K/V cache from device memory).  The key range is
 * cut into splits that run in parallel and are merged afterwards ("Q31：
 * FlashAttention 为什么快", follow-up 3), with the merge rule of the online
 * softmax ("GPU 学习日报 Day 21", section 5.2): partial results that share a reference max
 * add, others are rescaled by 2^(m_old - m_new) first.
 *
 * The work is a stream over K and V with ~1 FLOP per byte, so it runs on the
 * CUDA cores with wide coalesced loads; the tensor cores would add nothing.
 *
 *   decode_split_kernel   grid = B*H*S CTAs of 128 threads; CTA (head, split)
 *                         reads keys [s*L, min((s+1)*L, N)) once and writes an
 *                         unnormalised partial O (fp32, d values) plus its
 *                         (m, l) to the workspace.  Per warp, 32 keys at a
 *                         time: lane i owns key i for the dot product (16-byte
 *                         loads of its K row); the warp then walks the 32 keys,
 *                         broadcasting p_i, while each lane accumulates d/32
 *                         columns of p_i * v_i (coalesced 256-byte rows).
 *   decode_combine_kernel grid = B*H CTAs of d threads; merges the S partials,
 *                         divides by l, rounds O to bf16 and writes LSE.
 */
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <mutex>

#include "attn_fwd.h"

namespace {

constexpr int DEC_THREADS = 128;                 // 4 warps
constexpr int DEC_KEYS_PER_TILE = 32;            // one key per lane
constexpr int DEC_SPLIT_QUANTUM = 4 * DEC_KEYS_PER_TILE;
constexpr int64_t DEC_TARGET_CTAS = 8 * 148;     // a few waves of CTAs on a 148-SM part
constexpr float DEC_LN2 = 0.6931471805599453f;
constexpr float DEC_LOG2E = 1.4426950408889634f;

__device__ __forceinline__ float dec_ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

template <int D>
__global__ void __launch_bounds__(DEC_THREADS)
decode_split_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                    const __nv_bfloat16* __restrict__ v, float* __restrict__ part_o,
                    float2* __restrict__ part_ml, int N, int S, int L, float scale_log2) {
    constexpr int CPL = D / 32;                  // output columns per lane
    __shared__ float q_s[D];
    __shared__ float red_m[DEC_THREADS / 32];
    __shared__ float red_l[DEC_THREADS / 32];
    __shared__ float red_o[DEC_THREADS / 32][D];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t bh = blockIdx.x / S;
    const int s = blockIdx.x % S;
    const int begin = s * L;
    const int end = min(N, begin + L);
    const __nv_bfloat16* kh = k + bh * static_cast<int64_t>(N) * D;
    const __nv_bfloat16* vh = v + bh * static_cast<int64_t>(N) * D;

    for (int c = threadIdx.x; c < D; c += DEC_THREADS)
        q_s[c] = __bfloat162float(q[bh * D + c]) * scale_log2;   // scores in log2 units
    __syncthreads();

    float m_w = -INFINITY;       // warp-uniform reference max (log2 units)
    float l_lane = 0.0f;         // this lane's share of the row sum
    float acc[CPL];
#pragma unroll
    for (int e = 0; e < CPL; ++e) acc[e] = 0.0f;

    for (int t0 = begin + warp * DEC_KEYS_PER_TILE; t0 < end; t0 += DEC_THREADS) {
        const int key = t0 + lane;
        const bool valid = key < end;
        // score of this lane's key: 16-byte loads of its K row
        float sc = -INFINITY;
        if (valid) {
            const uint4* kr = reinterpret_cast<const uint4*>(kh + static_cast<int64_t>(key) * D);
            uint4 kv[D / 8];
#pragma unroll
            for (int u = 0; u < D / 8; ++u) kv[u] = __ldg(kr + u);
            float a0 = 0.0f, a1 = 0.0f;
#pragma unroll
            for (int u = 0; u < D / 8; ++u) {
                const uint32_t w[4] = {kv[u].x, kv[u].y, kv[u].z, kv[u].w};
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    a0 = fmaf(bf16_lo(w[h]), q_s[8 * u + 2 * h], a0);
                    a1 = fmaf(bf16_hi(w[h]), q_s[8 * u + 2 * h + 1], a1);
                }
            }
            sc = a0 + a1;
        }
        // online update with the tile max (t0 < end, so lane 0's key is valid)
        float mt = sc;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, off));
        const float m_new = fmaxf(m_w, mt);
        const float alpha = dec_ex2(m_w - m_new);            // 0 on the first tile
        const float p = valid ? dec_ex2(sc - m_new) : 0.0f;
        l_lane = l_lane * alpha + p;
#pragma unroll
        for (int e = 0; e < CPL; ++e) acc[e] *= alpha;
        m_w = m_new;
        // O += p_i v_i over the tile's keys; lane owns columns [CPL*lane, CPL*lane + CPL)
        const int nk = min(DEC_KEYS_PER_TILE, end - t0);
        const __nv_bfloat16* vt = vh + static_cast<int64_t>(t0) * D + CPL * lane;
#pragma unroll 8
        for (int i = 0; i < DEC_KEYS_PER_TILE; ++i) {
            const float pi = __shfl_sync(0xffffffffu, p, i);
            if (i < nk) {
                const __nv_bfloat16* vr = vt + static_cast<int64_t>(i) * D;
                if (CPL == 4) {
                    const uint2 w = __ldg(reinterpret_cast<const uint2*>(vr));
                    acc[0] = fmaf(pi, bf16_lo(w.x), acc[0]);
                    acc[1] = fmaf(pi, bf16_hi(w.x), acc[1]);
                    acc[2] = fmaf(pi, bf16_lo(w.y), acc[2]);
                    acc[3] = fmaf(pi, bf16_hi(w.y), acc[3]);
                } else {
                    const uint32_t w = __ldg(reinterpret_cast<const unsigned int*>(vr));
                    acc[0] = fmaf(pi, bf16_lo(w), acc[0]);
                    acc[1] = fmaf(pi, bf16_hi(w), acc[1]);
                }
            }
        }
    }

    // merge the warps: each warp's (m_w, l_w, acc) onto the CTA's reference max
    float l_w = l_lane;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) l_w += __shfl_xor_sync(0xffffffffu, l_w, off);
    if (lane == 0) {
        red_m[warp] = m_w;
        red_l[warp] = l_w;
    }
#pragma unroll
    for (int e = 0; e < CPL; ++e) red_o[warp][CPL * lane + e] = acc[e];
    __syncthreads();
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < DEC_THREADS / 32; ++w) M = fmaxf(M, red_m[w]);
    for (int c = threadIdx.x; c < D; c += DEC_THREADS) {
        float o = 0.0f;
#pragma unroll
        for (int w = 0; w < DEC_THREADS / 32; ++w)
            if (red_m[w] != -INFINITY) o += red_o[w][c] * dec_ex2(red_m[w] - M);
        part_o[(bh * S + s) * D + c] = o;
    }
    if (threadIdx.x == 0) {
        float Lsum = 0.0f;
#pragma unroll
        for (int w = 0; w < DEC_THREADS / 32; ++w)
            if (red_m[w] != -INFINITY) Lsum += red_l[w] * dec_ex2(red_m[w] - M);
        part_ml[bh * S + s] = make_float2(M, Lsum);
    }
}

template <int D>
__global__ void __launch_bounds__(D)
decode_combine_kernel(const float* __restrict__ part_o, const float2* __restrict__ part_ml,
                      __nv_bfloat16* __restrict__ o, float* __restrict__ lse, int S) {
    const int64_t bh = blockIdx.x;
    const int c = threadIdx.x;
    const float2* ml = part_ml + bh * S;
    float M = -INFINITY;
    for (int s = 0; s < S; ++s) M = fmaxf(M, ml[s].x);
    float Lsum = 0.0f, acc = 0.0f;
    for (int s = 0; s < S; ++s) {
        const float2 v = ml[s];
        if (v.x == -INFINITY) continue;
        const float w = dec_ex2(v.x - M);
        Lsum += v.y * w;
        acc += part_o[(bh * S + s) * D + c] * w;
    }
    o[bh * D + c] = __float2bfloat16_rn(Lsum > 0.0f ? acc / Lsum : 0.0f);
    if (c == 0) lse[bh] = (M + log2f(Lsum)) * DEC_LN2;
}

/* Split plan shared by the workspace query and the launch. */
struct DecodePlan {
    int S;   // splits per head
    int L;   // keys per split (a multiple of DEC_SPLIT_QUANTUM)
};

DecodePlan decode_plan(int64_t BH, int64_t N) {
    const int64_t max_splits = (N + DEC_SPLIT_QUANTUM - 1) / DEC_SPLIT_QUANTUM;
    int64_t S = (DEC_TARGET_CTAS + BH - 1) / BH;
    if (S > max_splits) S = max_splits;
    if (S < 1) S = 1;
    int64_t L = (N + S - 1) / S;
    L = (L + DEC_SPLIT_QUANTUM - 1) / DEC_SPLIT_QUANTUM * DEC_SPLIT_QUANTUM;
    S = (N + L - 1) / L;
    return DecodePlan{static_cast<int>(S), static_cast<int>(L)};
}

int decode_validate(int64_t B, int64_t H, int64_t N, int64_t d, float scale, bool* empty) {
    if (B < 0 || H < 0 || N < 0) return ATTN_ERR_SHAPE;
    if (d != 64 && d != 128) return ATTN_ERR_HEADDIM;
    if (!(scale > 0.0f) || !isfinite(scale)) return ATTN_ERR_SCALE;
    *empty = (B == 0 || H == 0 || N == 0);
    if (*empty) return ATTN_OK;
    if (N > INT32_MAX / 2 || H > INT32_MAX / B) return ATTN_ERR_SHAPE;
    const int64_t BH = B * H;
    if (BH * decode_plan(BH, N).S > INT32_MAX) return ATTN_ERR_SHAPE;
    return ATTN_OK;
}

size_t decode_ws_bytes(int64_t BH, int64_t N, int64_t d) {
    const DecodePlan pl = decode_plan(BH, N);
    const size_t po = static_cast<size_t>(BH) * pl.S * d * sizeof(float);
    return ((po + 255u) & ~static_cast<size_t>(255u)) +
           static_cast<size_t>(BH) * pl.S * sizeof(float2);
}

}  // namespace

extern "C" {

size_t attn_decode_workspace_bytes(int64_t B, int64_t H, int64_t N, int64_t d) {
    bool empty = false;
    if (decode_validate(B, H, N, d, 1.0f, &empty) != ATTN_OK) return 0;
    if (empty) return 0;
    return decode_ws_bytes(B * H, N, d);
}

int attn_decode(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B,
                int64_t H, int64_t N, int64_t d, float scale, void* workspace,
                size_t workspace_bytes, void* stream) {
    bool empty = false;
    int st = decode_validate(B, H, N, d, scale, &empty);
    if (st != ATTN_OK || empty) return st;
    if (!q || !k || !v || !o || !lse) return ATTN_ERR_NULL;
    const void* ptrs[5] = {q, k, v, o, lse};
    for (const void* ptr : ptrs)
        if (reinterpret_cast<uintptr_t>(ptr) & 15u) return ATTN_ERR_ALIGN;
    const int64_t BH = B * H;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
        workspace_bytes < decode_ws_bytes(BH, N, d))
        return ATTN_ERR_WORKSPACE;
    {
        // outputs (o, lse, the workspace) may not overlap the inputs or each other
        const uintptr_t qb0 = reinterpret_cast<uintptr_t>(q), kb0 = reinterpret_cast<uintptr_t>(k);
        const uintptr_t vb0 = reinterpret_cast<uintptr_t>(v);
        const uintptr_t out0[3] = {reinterpret_cast<uintptr_t>(o), reinterpret_cast<uintptr_t>(lse),
                                   reinterpret_cast<uintptr_t>(workspace)};
        const size_t outn[3] = {static_cast<size_t>(BH * d) * 2, static_cast<size_t>(BH) * 4,
                                decode_ws_bytes(BH, N, d)};
        const uintptr_t in0[3] = {qb0, kb0, vb0};
        const size_t inn[3] = {static_cast<size_t>(BH * d) * 2, static_cast<size_t>(BH * N * d) * 2,
                               static_cast<size_t>(BH * N * d) * 2};
        auto overlap = [](uintptr_t a, size_t na, uintptr_t b, size_t nb) { return a < b + nb && b < a + na; };
        for (int a = 0; a < 3; ++a) {
            for (int b = 0; b < 3; ++b)
                if (overlap(out0[a], outn[a], in0[b], inn[b])) return ATTN_ERR_OVERLAP;
            for (int b = a + 1; b < 3; ++b)
                if (overlap(out0[a], outn[a], out0[b], outn[b])) return ATTN_ERR_OVERLAP;
        }
    }
    int dev = 0, major = 0, minor = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
        cudaGetLastError();
        return ATTN_ERR_CUDA;
    }
    if (major != 10 || minor != 0) return ATTN_ERR_DEVICE;

    const DecodePlan pl = decode_plan(BH, N);
    const size_t po = static_cast<size_t>(BH) * pl.S * d * sizeof(float);
    float* part_o = static_cast<float*>(workspace);
    float2* part_ml = reinterpret_cast<float2*>(static_cast<char*>(workspace) +
                                                ((po + 255u) & ~static_cast<size_t>(255u)));
    const float sl = scale * DEC_LOG2E;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const auto* qb = static_cast<const __nv_bfloat16*>(q);
    const auto* kb = static_cast<const __nv_bfloat16*>(k);
    const auto* vb = static_cast<const __nv_bfloat16*>(v);
    auto* ob = static_cast<__nv_bfloat16*>(o);
    const unsigned grid = static_cast<unsigned>(BH * pl.S);
    if (d == 64) {
        decode_split_kernel<64><<<grid, DEC_THREADS, 0, s>>>(qb, kb, vb, part_o, part_ml,
                                                             static_cast<int>(N), pl.S, pl.L, sl);
        decode_combine_kernel<64><<<static_cast<unsigned>(BH), 64, 0, s>>>(part_o, part_ml, ob,
                                                                          lse, pl.S);
    } else {
        decode_split_kernel<128><<<grid, DEC_THREADS, 0, s>>>(qb, kb, vb, part_o, part_ml,
                                                              static_cast<int>(N), pl.S, pl.L, sl);
        decode_combine_kernel<128><<<static_cast<unsigned>(BH), 128, 0, s>>>(part_o, part_ml, ob,
                                                                            lse, pl.S);
    }
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_LAUNCH;
    return ATTN_OK;
}

}  // extern "C"

/*
 * Allocation-free decode.  Some callers cannot allocate device memory
 * themselves: a plugin or runtime whose host application owns all device
 * memory through its own pool, or a latency-bound loop that must not call
 * cudaMalloc (which can synchronise the device) once it is running.  For them
 * the per-split partial results live in this fixed buffer, part of the
 * library's own device image.  It is created with the module on every GPU
 * that loads the library and stays until the process exits.
 */
constexpr size_t DECODE_STATIC_SCRATCH_BYTES = size_t(8) << 20;   // 8 MiB
static __device__ __align__(256) unsigned char g_decode_scratch[DECODE_STATIC_SCRATCH_BYTES];

namespace {
constexpr int SCRATCH_MAX_DEVICES = 64;
std::mutex g_scratch_mutex;
void* g_scratch_ptr[SCRATCH_MAX_DEVICES] = {};

/* Device address of g_decode_scratch on the current device.  In host code the
 * array's name only stands in for the symbol, so the address is looked up once
 * per device (with that device current) and cached. */
int scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) { cudaGetLastError(); return ATTN_ERR_CUDA; }
    if (dev < 0 || dev >= SCRATCH_MAX_DEVICES) return ATTN_ERR_DEVICE;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_scratch_ptr[dev]) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_decode_scratch) != cudaSuccess || !ptr) {
            cudaGetLastError();
            return ATTN_ERR_CUDA;
        }
        g_scratch_ptr[dev] = ptr;
    }
    *out = g_scratch_ptr[dev];
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
    if (decode_ws_bytes(B * H, N, d) > DECODE_STATIC_SCRATCH_BYTES) return ATTN_ERR_WORKSPACE;
    void* scratch = nullptr;
    if ((st = scratch_address(&scratch)) != ATTN_OK) return st;
    return attn_decode(q, k, v, o, lse, B, H, N, d, scale, scratch, DECODE_STATIC_SCRATCH_BYTES,
                       stream);
}

}  // extern "C"
