/*
 * attn_fwd_sm100.cu -- fused exact-attention forward for B200 (sm_100a) and
 * the C ABI around it.
 *
 * What is computed (FlashAttention teaching pages): per head,
 *   O = softmax(scale * Q K^T [+ causal mask]) V  and  LSE_i = ln sum_j e^{s_ij}
 * ("GPU 学习日报 Day 21", sections 3.1 and 5.3; the saved statistic of airsota
 * "science-depth-m4-047", section 3 point (c)).  The N x N matrices S and P
 * exist only tile by tile on chip ("GPU 学习日报 Day 21", section 4): S in
 * tensor memory (TMEM), P overwriting S in TMEM as bf16, never in device memory.
 *
 * How it maps onto sm_100a (one persistent CTA per SM, 12 warps in three
 * warpgroups; setmaxnreg gives the two softmax warpgroups 208 registers per
 * thread and the third, which holds the TMA and MMA warps, 88):
 *   warp 8      TMA producer: Q tiles once per work unit, then K_j, V_j through
 *               a ring of shared-memory stages guarded by mbarriers.
 *   warp 9      MMA issuer (one thread): tcgen05.mma S_t = Q_t K_j^T into TMEM
 *               (both operands in shared memory), then O_t += P_t V_j with P_t
 *               read from TMEM and V_j from shared memory.  It also owns the
 *               TMEM allocation (512 columns).
 *   warps 10-11 no role (they complete the third warpgroup).
 *   warps 0-3   softmax for Q tile 0; warps 4-7 softmax for Q tile 1.  Thread
 *               r owns row r of its tile, which is TMEM lane r, so the row max
 *               and row sum need no shuffles.  Online recurrence of "GPU 学习日报
 *               Day 21", section 5.3, in base 2 with log2(e) folded into the scale,
 *               with lazy rescaling: the reference max only moves when a block
 *               max exceeds it by more than lazy_tau (so 2^{c s - m} <= 2^tau), which is
 *               exact because numerator and denominator share the reference
 *               (the same page, section 5.2).  At the end of a unit the same warps
 *               divide O by l, round to bf16 and store O and LSE.
 *   A work unit is a pair of 128-row Q tiles of one head; the two tiles share
 *   every K/V block and ping-pong on the tensor core (while one tile's softmax
 *   runs, the other tile's GEMMs run).  Causal: blocks above the diagonal are
 *   never loaded or computed; only the diagonal block is masked element-wise
 *   (the same page, section 6 table).  Causal units are grouped into mirror
 *   pairs of equal total length, which keeps the persistent CTAs in step on a
 *   few heads at a time (K/V read from HBM about once), and the last round's
 *   worth is dealt longest first (see sched_unit).
 *
 * Every wait on an mbarrier is bounded (iterations and wall time); when one
 * runs out the CTA records ATTN_ERR_TIMEOUT in a device status word, raises an
 * abort flag that the other warps see, waits (bounded) for its own copies and
 * MMAs in flight, frees its TMEM and exits.
 */
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <mutex>

#include "attn_fwd.h"

#define ATTN_VERSION "0.1.0"

namespace {

/* ------------------------------------------------------------------------ */
/* Tile configuration                                                        */
/* ------------------------------------------------------------------------ */
constexpr int BLOCK_M = 128;          // query rows per Q tile = TMEM lanes
constexpr int BLOCK_N = 128;          // key/value rows per K/V block
constexpr int UNIT_ROWS = 2 * BLOCK_M;  // a work unit = two Q tiles
constexpr int NUM_THREADS = 384;      // 3 warpgroups: softmax tile 0, softmax tile 1, TMA + MMA
/* Register split (setmaxnreg): the kernel launches with 168 registers per
 * thread (384 x 168 = 64512); the producer/MMA warpgroup gives back down to
 * 88 so that the two softmax warpgroups can hold 208: 2*128*208 + 128*88 =
 * 64512, exactly what the launch holds (a larger sum would wait forever). */
constexpr int LAUNCH_REGS = 168;      // per thread at launch (checked on the host before launching)
constexpr int SOFTMAX_REGS = 208;
constexpr int OTHER_REGS = 88;
static_assert(2 * 128 * SOFTMAX_REGS + 128 * OTHER_REGS == NUM_THREADS * LAUNCH_REGS, "register split");
constexpr int LOAD_WARP = 8;
constexpr int MMA_WARP = 9;
constexpr int TMEM_COLS = 512;
constexpr int CHUNK_ELEMS = 64;                     // one 128-byte swizzle atom of bf16
constexpr int CHUNK_BYTES = BLOCK_M * 128;          // 128 rows x 128 bytes
/* Lazy-rescale threshold, log2 units: the reference max moves only when a
 * block max exceeds it by more than TAU, so p = 2^(c s - m_ref) <= 2^TAU.
 * bf16 P: TAU = 32, so a row sum stays below 2^32 * N < 2^63, far inside fp32,
 * and every value keeps its relative precision; a larger TAU means fewer O
 * rescales (measured +2.5 % on peaked logits against TAU = 8, no change
 * elsewhere).  e4m3 P saturates at 448, so there TAU = 8 (p <= 256). */
template <bool FP8>
__device__ __forceinline__ constexpr float lazy_tau() { return FP8 ? 8.0f : 32.0f; }
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;   // 2 s: a correct run never waits 1 ms
constexpr uint64_t TEST_WAIT_LIMIT_NS = 20000000ull; // 20 ms, for the timeout test hook
constexpr uint32_t WAIT_MAX_ITERS = 1u << 28;
constexpr float LN2 = 0.6931471805599453f;
constexpr float LOG2E = 1.4426950408889634f;

/* FP8: e4m3 Q, K, V, V read transposed (d rows, keys contiguous) so that every
 * operand is K-major.  A Q or K row is one 128-byte swizzle atom at d = 128 and
 * a 64-byte one at d = 64; a V^T row (128 keys of one block) is 128 bytes. */
template <int D, bool FP8 = false>
struct Cfg {
    static constexpr int TILE_BYTES = BLOCK_M * D * (FP8 ? 1 : 2);   // 128 rows x D elements
    static constexpr int CHUNKS = FP8 ? 1 : D / CHUNK_ELEMS;          // swizzle atoms along d
    static constexpr int NSTAGE = (FP8 || D == 64) ? 4 : 2;  // ring stages, each K_j then V_j
    static constexpr int Q_OFF = 0;
    static constexpr int RING_OFF = 2 * TILE_BYTES;
    static constexpr int BAR_OFF = RING_OFF + 2 * NSTAGE * TILE_BYTES;
    static constexpr int NUM_BARS = 2 + 2 * NSTAGE + 8 + 1;
    static constexpr int MISC_OFF = BAR_OFF + 8 * NUM_BARS;
    static constexpr int SMEM_BYTES = MISC_OFF + 16 + 1024;  // + alignment slack
    // TMEM columns: S/P of tile t at 128*t, O of tile t at 256 + D*t
    static constexpr uint32_t S_COL0 = 0, S_COL1 = 128;
    static constexpr uint32_t O_COL0 = 256, O_COL1 = 256 + D;
    static_assert(D == 64 || D == 128, "head dim");
    // Q and K rows of e4m3 at d = 64 are 64 bytes: 64-byte swizzle (TMA and MMA)
    static constexpr bool QK_SW64 = FP8 && D == 64;
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
};

struct FwdParams {
    __nv_bfloat16* o;
    float* lse;
    int N;          // sequence length
    int BH;         // B * H
    int n_pairs;    // ceil(N / 256)
    int nkv;        // ceil(N / 128)
    int n_units;    // BH * n_pairs
    float scale_log2;  // scale * log2(e)
    uint64_t wait_limit_ns;  // bound on every mbarrier wait
    int withhold_kv;         // test hook: the producer never loads K/V, so waits run out
    float o_scale;           // e4m3 path: V's descale factor, applied to O at the end
    /* causal schedule (plan_schedule): mirror-job rounds, then the tail */
    int jobs_per_head;       // ceil(n_pairs / 2)
    int mirror_rounds;       // rounds of one mirror job per CTA
    int tail_bh0;            // first head with units in the tail
    int tail_m0;             // jobs of head tail_bh0 below this index ran as mirror jobs
    int tail_full;           // heads after tail_bh0 (all their units are in the tail)
    int tail_a;              // tail units of the top tail_m0 pair indices
    int tail_b;              // tail units of the middle pair indices (tail_bh0 included)
    int tail_units;          // all tail units
};

__device__ int g_attn_status = 0;

/* ------------------------------------------------------------------------ */
/* PTX wrappers                                                              */
/* ------------------------------------------------------------------------ */
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void record_error(int code) { atomicCAS(&g_attn_status, 0, code); }

/* Slow path of mbar_wait (inlined into kernels that change their register
 * budget with setmaxnreg, which cannot make calls; a call elsewhere). */
__device__ __forceinline__ bool mbar_wait_slow_body(uint32_t bar, uint32_t parity,
                                                    volatile uint32_t* abort_flag, uint64_t limit_ns) {
    const uint64_t t0 = globaltimer();
    for (uint32_t it = 0; it < WAIT_MAX_ITERS; ++it) {
        if (mbar_try(bar, parity)) return true;
        if ((it & 63u) == 63u) {
            if (*abort_flag) return false;
            if (globaltimer() - t0 > limit_ns) break;
        }
    }
    record_error(ATTN_ERR_TIMEOUT);
    *abort_flag = 1u;
    return false;
}

__device__ __noinline__ bool mbar_wait_slow(uint32_t bar, uint32_t parity, volatile uint32_t* abort_flag,
                                            uint64_t limit_ns) {
    return mbar_wait_slow_body(bar, parity, abort_flag, limit_ns);
}

/* Bounded wait for the phase of parity `parity` of an mbarrier.  Returns false
 * when another warp raised the abort flag, or after the limit (then it records
 * the timeout and raises the flag itself). */
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile uint32_t* abort_flag,
                                          uint64_t limit_ns) {
    if (mbar_try(bar, parity)) return true;
    return mbar_wait_slow(bar, parity, abort_flag, limit_ns);
}

/* The same, with no call (for the setmaxnreg kernel). */
__device__ __forceinline__ bool mbar_wait_inl(uint32_t bar, uint32_t parity, volatile uint32_t* abort_flag,
                                              uint64_t limit_ns) {
    if (mbar_try(bar, parity)) return true;
    return mbar_wait_slow_body(bar, parity, abort_flag, limit_ns);
}

/* Bounded wait that ignores the abort flag: used on the abort path to let the
 * CTA's own copies and MMAs in flight land before it exits. */
__device__ __forceinline__ void mbar_drain_wait_inl(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
    const uint64_t t0 = globaltimer();
    for (uint32_t it = 0; it < WAIT_MAX_ITERS; ++it) {
        if (mbar_try(bar, parity)) return;
        if ((it & 63u) == 63u && globaltimer() - t0 > limit_ns) return;
    }
}

__device__ __noinline__ void mbar_drain_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
    mbar_drain_wait_inl(bar, parity, limit_ns);
}

__device__ __forceinline__ void tma_load_3d(const CUtensorMap* map, uint32_t dst, uint32_t bar,
                                            int c0, int c1, int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

/* Shared-memory matrix descriptor for tcgen05.mma, 128-byte swizzle.
 * Bits: [0,14) start >> 4, [16,30) leading byte offset >> 4, [32,46) stride
 * byte offset >> 4, [46,48) version (1 on sm_100), [61,64) layout (2 = 128B swizzle). */
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
    d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
    d |= static_cast<uint64_t>(1) << 46;
    d |= static_cast<uint64_t>(2) << 61;
    return d;
}

/* The same descriptor with 64-byte swizzle ([61,64) = 4): rows of 64 bytes,
 * 8-row groups 512 bytes apart. */
__device__ __forceinline__ uint64_t sdesc_sw64(uint32_t saddr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>(1) << 16;                      // leading byte offset (unused here)
    d |= static_cast<uint64_t>((512u >> 4) & 0x3FFFu) << 32;  // stride byte offset
    d |= static_cast<uint64_t>(1) << 46;
    d |= static_cast<uint64_t>(4) << 61;
    return d;
}

/* Instruction descriptor, kind::f16: bf16 x bf16 -> fp32, dense.
 * Bits: [4,6) D format (1 = f32), [7,10) A format (1 = bf16), [10,13) B format,
 * 15 A major (0 = K), 16 B major (1 = MN), [17,23) N >> 3, [24,29) M >> 4. */
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) |
           (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

/* The MMA statements carry no memory clobber: they touch no memory the compiler
 * tracks, and as volatile asm they stay ordered with the (clobbering) waits,
 * fences and commits around them. */
/* `leader` selects the one thread that issues: the MMA warp runs its loop with
 * all 32 lanes (so the descriptor arithmetic is warp-uniform) and lane 0
 * issues every MMA and every commit (a commit tracks the MMAs of the thread
 * that issues it). */
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate, uint32_t leader = 1u) {
    asm volatile(
        "{\n\t.reg .pred p, e;\n\tsetp.ne.b32 p, %4, 0;\n\tsetp.ne.b32 e, %5, 0;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(leader));
}

__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate, uint32_t leader = 1u) {
    asm volatile(
        "{\n\t.reg .pred p, e;\n\tsetp.ne.b32 p, %4, 0;\n\tsetp.ne.b32 e, %5, 0;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
        ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(leader));
}

__device__ __forceinline__ void mma_commit(uint32_t bar, uint32_t leader = 1u) {
    asm volatile("{\n\t.reg .pred e;\n\tsetp.ne.b32 e, %1, 0;\n\t"
                 "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}"
                 ::"r"(bar), "r"(leader)
                 : "memory");
}

/* S = Q K^T for one 128x128 tile: D/16 MMAs with K = 16.  a0 / b0 describe
 * the first 16 columns of Q and K; k-step kk starts (kk/4) swizzle atoms plus
 * (kk%4)*32 bytes further, which only moves the start-address field. */
template <int D>
__device__ __forceinline__ void issue_qk(uint32_t d_tmem, uint64_t a0, uint64_t b0, uint32_t idesc,
                                         uint32_t leader = 1u) {
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        const uint64_t off = static_cast<uint64_t>(((kk >> 2) * CHUNK_BYTES + (kk & 3) * 32) >> 4);
        mma_ss(d_tmem, a0 + off, b0 + off, idesc, kk > 0 ? 1u : 0u, leader);
    }
}

/* O += P V for keys [64*half, 64*half + 64) of one block: 4 MMAs with K = 16.
 * P is bf16 in TMEM (keys 2c, 2c+1 in column c); b0 describes V's first 16
 * keys (MN-major: 16 keys = 2048 bytes further per k-step). */
__device__ __forceinline__ void issue_pv_half(uint32_t d_tmem, uint32_t p_tmem, uint64_t b0,
                                              uint32_t idesc, uint32_t acc_first, int half,
                                              uint32_t leader) {
#pragma unroll
    for (int i = 0; i < BLOCK_N / 32; ++i) {
        const int kk = half * (BLOCK_N / 32) + i;
        const uint64_t off = static_cast<uint64_t>((kk * 16 * 128) >> 4);
        mma_ts(d_tmem, p_tmem + kk * 8, b0 + off, idesc, (i > 0) ? 1u : acc_first, leader);
    }
}

/* e4m3 x e4m3 -> fp32 (kind::f8f6f4), dense, both operands K-major.
 * Bits: [4,6) D format (1 = f32), [7,10) / [10,13) A / B format (0 = E4M3),
 * 15 / 16 majors (0 = K), [17,23) N >> 3, [24,29) M >> 4. */
__host__ __device__ constexpr uint32_t idesc_e4m3(int M, int N) {
    return (1u << 4) | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void mma_ss_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate, uint32_t leader) {
    asm volatile(
        "{\n\t.reg .pred p, e;\n\tsetp.ne.b32 p, %4, 0;\n\tsetp.ne.b32 e, %5, 0;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(leader));
}

__device__ __forceinline__ void mma_ts_f8(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate, uint32_t leader) {
    asm volatile(
        "{\n\t.reg .pred p, e;\n\tsetp.ne.b32 p, %4, 0;\n\tsetp.ne.b32 e, %5, 0;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}"
        ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(leader));
}

/* S = Q K^T with e4m3 Q and K (a row of D bytes is one swizzle atom, 128- or
 * 64-byte): D / 32 MMAs with K = 32, each starting 32 bytes further. */
template <int D>
__device__ __forceinline__ void issue_qk_f8(uint32_t d_tmem, uint64_t a0, uint64_t b0, uint32_t idesc,
                                            uint32_t leader) {
#pragma unroll
    for (int kk = 0; kk < D / 32; ++kk) {
        const uint64_t off = static_cast<uint64_t>((kk * 32) >> 4);
        mma_ss_f8(d_tmem, a0 + off, b0 + off, idesc, kk > 0 ? 1u : 0u, leader);
    }
}

/* O += P V for keys [64*half, 64*half + 64) with e4m3 P and V: 2 MMAs with
 * K = 32.  P is in TMEM (keys 4c .. 4c+3 in column c, key 4c in bits 0-7); b0
 * describes V^T (d rows, keys contiguous: K-major), 32 keys = 32 bytes further
 * per k-step. */
__device__ __forceinline__ void issue_pv_half_f8(uint32_t d_tmem, uint32_t p_tmem, uint64_t b0,
                                                 uint32_t idesc, uint32_t acc_first, int half,
                                                 uint32_t leader) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int kk = half * 2 + i;
        mma_ts_f8(d_tmem, p_tmem + kk * 8, b0 + static_cast<uint64_t>((kk * 32) >> 4), idesc,
                  (i > 0) ? 1u : acc_first, leader);
    }
}

template <int D, bool FP8>
__device__ __forceinline__ void issue_s(uint32_t d_tmem, uint64_t a0, uint64_t b0, uint32_t idesc,
                                        uint32_t leader) {
    if constexpr (FP8) issue_qk_f8<D>(d_tmem, a0, b0, idesc, leader);
    else issue_qk<D>(d_tmem, a0, b0, idesc, leader);
}

template <bool FP8>
__device__ __forceinline__ void issue_pv(uint32_t d_tmem, uint32_t p_tmem, uint64_t b0,
                                         uint32_t idesc, uint32_t acc_first, int half,
                                         uint32_t leader) {
    if constexpr (FP8) issue_pv_half_f8(d_tmem, p_tmem, b0, idesc, acc_first, half, leader);
    else issue_pv_half(d_tmem, p_tmem, b0, idesc, acc_first, half, leader);
}

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float fmax3f(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

/* Packed pairs of fp32 (one 64-bit register pair) for the sm_100 f32x2 pipes. */
__device__ __forceinline__ uint64_t f2pack(float a, float b) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ void f2unpack(uint64_t v, float& a, float& b) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

__device__ __forceinline__ uint64_t fsub2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

/* 2^x for a pair of values on the FMA/ALU pipes, to relieve the MUFU unit.
 * Range reduction (Cody-Waite style): x = n + f with n = round(x), obtained by
 * adding and subtracting 1.5 * 2^23 in fp32, and f in [-1/2, 1/2].  2^f is the
 * degree-3 polynomial with minimax relative error on [-1/2, 1/2], from a Remez
 * exchange in fp64 with the coefficients rounded to fp32: max relative error
 * 7.5e-5 over the fp32 evaluation, far below the bf16 rounding of P (a CPU test
 * re-evaluates this arithmetic and checks the bound).  2^n is applied by
 * adding n to the exponent field: the low mantissa bits of x + 1.5 * 2^23 hold
 * n, so shifting its bit pattern left by 23 yields n << 23.  x is clamped at
 * -125 so the exponent stays normal (2^-125 is negligible next to a row whose
 * largest term is >= 1). */
constexpr float EXP2_ROUND = 12582912.0f;          // 1.5 * 2^23
constexpr float EXP2_C0 = 9.999280572e-01f;
constexpr float EXP2_C1 = 6.932609677e-01f;
constexpr float EXP2_C2 = 2.426111251e-01f;
constexpr float EXP2_C3 = 5.517166853e-02f;

__device__ __forceinline__ void exp2_poly_pair(float x0, float x1, float& p0, float& p1) {
    const uint64_t x = f2pack(fmaxf(x0, -125.0f), fmaxf(x1, -125.0f));
    const uint64_t rnd = f2pack(EXP2_ROUND, EXP2_ROUND);
    const uint64_t t = fadd2(x, rnd);
    const uint64_t f = fsub2(x, fsub2(t, rnd));
    uint64_t q = ffma2(f2pack(EXP2_C3, EXP2_C3), f, f2pack(EXP2_C2, EXP2_C2));
    q = ffma2(q, f, f2pack(EXP2_C1, EXP2_C1));
    q = ffma2(q, f, f2pack(EXP2_C0, EXP2_C0));
    float q0, q1, t0, t1;
    f2unpack(q, q0, q1);
    f2unpack(t, t0, t1);
    p0 = __int_as_float(__float_as_int(q0) + (__float_as_int(t0) << 23));
    p1 = __int_as_float(__float_as_int(q1) + (__float_as_int(t1) << 23));
}

/* Which column pairs of a score row take the polynomial (bit k%8 of the mask
 * for pair k); the rest use the MUFU ex2.  2 of 8 pairs on the FMA pipe where
 * the exponentials outweigh the tensor work per block: bf16 at d = 64 (+2.3 %)
 * and e4m3 at both head dimensions (+8.7 % on causal N = 8192 d = 128, +5.8 %
 * on N = 2048 d = 64; 1/8 gains half of that, 4/8 and 5/8 lose).  For bf16 at
 * d = 128, where MUFU and tensor work per block are equal, every fraction
 * measured was slower than or equal to none. */
template <int D, bool FP8>
__device__ __forceinline__ constexpr uint32_t exp2_poly_mask() {
    return (D == 64 || FP8) ? 0x11u : 0x00u;
}

/* Two fp32 -> one bf16x2 word, round to nearest even; `lo` in bits 0-15. */
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

/* Four fp32 -> four e4m3 in one word, round to nearest even, saturating at
 * +-448; `a` in bits 0-7.  (cvt ... e4m3x2 d, x, y puts x in the upper byte.) */
__device__ __forceinline__ uint32_t pack_e4m3x4(float a, float b, float c, float d) {
    uint32_t r;
    asm("{\n\t.reg .b16 lo, hi;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 lo, %2, %1;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 hi, %4, %3;\n\t"
        "mov.b32 %0, {lo, hi};\n\t}"
        : "=r"(r) : "f"(a), "f"(b), "f"(c), "f"(d));
    return r;
}

/* tcgen05.ld of 128 consecutive 32-bit columns of this thread's TMEM lane, with
 * the wait in the same asm statement so no use of v[] can be scheduled early. */
__device__ __forceinline__ void tmem_ld128_wait(uint32_t taddr, uint32_t* v) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x128.b32 {"
        "%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, "
        "%32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, "
        "%48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63, "
        "%64, %65, %66, %67, %68, %69, %70, %71, %72, %73, %74, %75, %76, %77, %78, %79, "
        "%80, %81, %82, %83, %84, %85, %86, %87, %88, %89, %90, %91, %92, %93, %94, %95, "
        "%96, %97, %98, %99, %100, %101, %102, %103, %104, %105, %106, %107, %108, %109, %110, %111, "
        "%112, %113, %114, %115, %116, %117, %118, %119, %120, %121, %122, %123, %124, %125, %126, %127"
        "}, [%128];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
          "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
          "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31]),
          "=r"(v[32]), "=r"(v[33]), "=r"(v[34]), "=r"(v[35]), "=r"(v[36]), "=r"(v[37]), "=r"(v[38]), "=r"(v[39]),
          "=r"(v[40]), "=r"(v[41]), "=r"(v[42]), "=r"(v[43]), "=r"(v[44]), "=r"(v[45]), "=r"(v[46]), "=r"(v[47]),
          "=r"(v[48]), "=r"(v[49]), "=r"(v[50]), "=r"(v[51]), "=r"(v[52]), "=r"(v[53]), "=r"(v[54]), "=r"(v[55]),
          "=r"(v[56]), "=r"(v[57]), "=r"(v[58]), "=r"(v[59]), "=r"(v[60]), "=r"(v[61]), "=r"(v[62]), "=r"(v[63]),
          "=r"(v[64]), "=r"(v[65]), "=r"(v[66]), "=r"(v[67]), "=r"(v[68]), "=r"(v[69]), "=r"(v[70]), "=r"(v[71]),
          "=r"(v[72]), "=r"(v[73]), "=r"(v[74]), "=r"(v[75]), "=r"(v[76]), "=r"(v[77]), "=r"(v[78]), "=r"(v[79]),
          "=r"(v[80]), "=r"(v[81]), "=r"(v[82]), "=r"(v[83]), "=r"(v[84]), "=r"(v[85]), "=r"(v[86]), "=r"(v[87]),
          "=r"(v[88]), "=r"(v[89]), "=r"(v[90]), "=r"(v[91]), "=r"(v[92]), "=r"(v[93]), "=r"(v[94]), "=r"(v[95]),
          "=r"(v[96]), "=r"(v[97]), "=r"(v[98]), "=r"(v[99]), "=r"(v[100]), "=r"(v[101]), "=r"(v[102]), "=r"(v[103]),
          "=r"(v[104]), "=r"(v[105]), "=r"(v[106]), "=r"(v[107]), "=r"(v[108]), "=r"(v[109]), "=r"(v[110]), "=r"(v[111]),
          "=r"(v[112]), "=r"(v[113]), "=r"(v[114]), "=r"(v[115]), "=r"(v[116]), "=r"(v[117]), "=r"(v[118]), "=r"(v[119]),
          "=r"(v[120]), "=r"(v[121]), "=r"(v[122]), "=r"(v[123]), "=r"(v[124]), "=r"(v[125]), "=r"(v[126]), "=r"(v[127])
        : "r"(taddr)
        : "memory");
}

/* tcgen05.ld of 32 consecutive 32-bit columns of this thread's TMEM lane, with
 * the wait in the same asm statement so no use of v[] can be scheduled early. */
__device__ __forceinline__ void tmem_ld32_wait(uint32_t taddr, uint32_t* v) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {"
        "%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31"
        "}, [%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
          "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
          "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
        : "r"(taddr)
        : "memory");
}

/* tcgen05.st of 32 consecutive 32-bit columns into this thread's TMEM lane. */
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* v) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {"
        "%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
        "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32"
        "};"
        :
        : "r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
          "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]),
          "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]),
          "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
}

/* tcgen05.st of 16 consecutive 32-bit columns into this thread's TMEM lane. */
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* v) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {"
        "%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16"
        "};"
        :
        : "r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]),
          "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]),
          "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}

/* tcgen05.st of 8 consecutive 32-bit columns into this thread's TMEM lane. */
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t* v) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};"
        :
        : "r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]),
          "r"(v[6]), "r"(v[7])
        : "memory");
}

__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

/* ------------------------------------------------------------------------ */
/* Work units and the static schedule                                        */
/* ------------------------------------------------------------------------ */
struct Unit {
    int bh;     // flat head index b*H + h
    int pair;   // Q rows [256*pair, 256*pair + 256)
    int n[2];   // K/V blocks Q tile t needs (0 when the tile lies past N)
};

__host__ __device__ __forceinline__ void fill_unit(Unit& u, bool causal, const FwdParams& p) {
#pragma unroll
    for (int t = 0; t < 2; ++t) {
        const int r0 = u.pair * UNIT_ROWS + t * BLOCK_M;
        if (r0 >= p.N) {
            u.n[t] = 0;
        } else if (causal) {
            const int last = r0 / BLOCK_N;          // the diagonal block of this tile
            u.n[t] = last + 1 < p.nkv ? last + 1 : p.nkv;
        } else {
            u.n[t] = p.nkv;
        }
    }
}

/* The s-th work unit of CTA `cta` out of `grid`.  Returns 1 with u filled, 0
 * for an empty slot (skip it), -1 past the CTA's last unit.  Every warp role of
 * a CTA walks the same sequence.
 *
 * Non-causal: every unit has the same work; units go round-robin in head-major
 * order, so the CTAs of a round share the K/V of a few heads in L2.
 *
 * Causal (units need 2*pair + 1 and 2*pair + 2 K/V blocks for their two Q
 * tiles, so they differ in length): a job is the mirror pair of units
 * {P-1-m, m} of one head (P = n_pairs).  Its two units need
 * 2(P-1-m) + 2 + 2m + 2 = 2P + 2 blocks in all, the same for every job, so in
 * each of the first mirror_rounds rounds every CTA runs one job and all CTAs
 * stay in step; the jobs of one round are those of a few consecutive heads, so
 * each head's K/V blocks come from HBM once and then from L2.  The remaining
 * units (at least one round's worth of jobs) are ordered longest first
 * (pair index descending, head ascending) and dealt in snake order (round r
 * gives CTA c the unit r*G + c when r is even, r*G + G-1-c when odd), which
 * evens out the end of the launch.  plan_schedule sets the parameters. */
__host__ __device__ __forceinline__ int sched_unit(int s, int cta, int grid, bool causal,
                                                   const FwdParams& p, Unit& u) {
    if (!causal) {
        const int idx = s * grid + cta;
        if (idx >= p.n_units) return -1;
        u.bh = idx / p.n_pairs;
        u.pair = idx - u.bh * p.n_pairs;
        fill_unit(u, false, p);
        return 1;
    }
    const int P = p.n_pairs;
    if (s < 2 * p.mirror_rounds) {
        const int job = (s >> 1) * grid + cta;
        u.bh = job / p.jobs_per_head;
        const int m = job - u.bh * p.jobs_per_head;
        if (s & 1) {
            if (2 * m == P - 1) return 0;       // the middle unit of an odd P stands alone
            u.pair = m;
        } else {
            u.pair = P - 1 - m;
        }
    } else {
        const int r = s - 2 * p.mirror_rounds;
        const int i = r * grid + ((r & 1) ? (grid - 1 - cta) : cta);
        if (i >= p.tail_units) return -1;
        const int hf = p.tail_full, m0 = p.tail_m0, bh0 = p.tail_bh0;
        if (i < p.tail_a) {                           // pairs P-1 .. P-m0: full heads only
            u.pair = P - 1 - i / hf;
            u.bh = bh0 + 1 + i % hf;
        } else if (i < p.tail_a + p.tail_b) {         // pairs P-1-m0 .. m0: head bh0 too
            const int k = i - p.tail_a;
            u.pair = P - 1 - m0 - k / (hf + 1);
            u.bh = bh0 + k % (hf + 1);
        } else {                                      // pairs m0-1 .. 0: full heads only
            const int k = i - p.tail_a - p.tail_b;
            u.pair = m0 - 1 - k / hf;
            u.bh = bh0 + 1 + k % hf;
        }
    }
    fill_unit(u, true, p);
    return 1;
}

/* Host side of the causal schedule: mirror rounds leave at least one round of
 * jobs to the longest-first tail. */
inline void plan_schedule(FwdParams& p, int grid) {
    const int P = p.n_pairs;
    p.jobs_per_head = (P + 1) / 2;
    const int64_t njobs = static_cast<int64_t>(p.BH) * p.jobs_per_head;
    const int64_t rounds = njobs / grid - 1;
    p.mirror_rounds = rounds > 0 ? static_cast<int>(rounds) : 0;
    const int64_t first = static_cast<int64_t>(p.mirror_rounds) * grid;   // first tail job
    p.tail_bh0 = static_cast<int>(first / p.jobs_per_head);
    p.tail_m0 = static_cast<int>(first % p.jobs_per_head);
    p.tail_full = p.BH - 1 - p.tail_bh0;
    p.tail_a = p.tail_m0 * p.tail_full;
    p.tail_b = (P - 2 * p.tail_m0) * (p.tail_full + 1);
    p.tail_units = 2 * p.tail_a + p.tail_b;
}

/* ------------------------------------------------------------------------ */
/* The kernel                                                                */
/* ------------------------------------------------------------------------ */
template <int D, bool CAUSAL, bool FP8 = false>
__global__ void __launch_bounds__(NUM_THREADS, 1)
attn_fwd_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
    using C = Cfg<D, FP8>;
    constexpr int NSTAGE = C::NSTAGE;
    constexpr uint32_t TILE = C::TILE_BYTES;

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;   // 128B swizzle needs 1024B-aligned tiles
    uint8_t* const base_ptr = smem_raw + (base - raw);

    const uint32_t sQ[2] = {base + C::Q_OFF, base + C::Q_OFF + TILE};
    const uint32_t sRing = base + C::RING_OFF;
    const uint32_t bars = base + C::BAR_OFF;
    const uint32_t bar_q_full = bars;
    const uint32_t bar_q_empty = bars + 8;
    auto bar_kv_full = [&](int s) { return bars + 16 + 8u * s; };
    auto bar_kv_empty = [&](int s) { return bars + 16 + 8u * (NSTAGE + s); };
    const uint32_t bar_s_full0 = bars + 16 + 16 * NSTAGE;      // [2]
    const uint32_t bar_p_ready0 = bar_s_full0 + 16;            // [2]
    const uint32_t bar_o_full0 = bar_p_ready0 + 16;            // [2]
    const uint32_t bar_p_half0 = bar_o_full0 + 16;             // [2]
    const uint32_t bar_drain = bar_p_half0 + 16;
    uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + C::MISC_OFF);
    volatile uint32_t* const abort_flag = reinterpret_cast<volatile uint32_t*>(base_ptr + C::MISC_OFF + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint64_t wlim = p.wait_limit_ns;

    if (threadIdx.x == 0) {
        mbar_init(bar_q_full, 1);
        mbar_init(bar_q_empty, 1);
        for (int s = 0; s < NSTAGE; ++s) {
            mbar_init(bar_kv_full(s), 1);
            mbar_init(bar_kv_empty(s), 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(bar_s_full0 + 8 * t, 1);
            mbar_init(bar_p_ready0 + 8 * t, BLOCK_M);   // every softmax thread of the tile
            mbar_init(bar_o_full0 + 8 * t, 1);
            mbar_init(bar_p_half0 + 8 * t, BLOCK_M);    // first half of P_t stored
        }
        mbar_init(bar_drain, 1);
        *abort_flag = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == LOAD_WARP && lane == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
    }
    if (warp == MMA_WARP) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(tmem_slot)), "r"(TMEM_COLS) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == LOAD_WARP) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(OTHER_REGS) : "memory");
        /* ---------------- TMA producer ---------------- */
        if (lane == 0) {
            uint32_t it = 0;          // K/V ring position (K_j and V_j each take one)
            int local = 0;            // units this CTA has started
            bool aborted = false;
            for (int r = 0;; ++r) {
                Unit u;
                const int got = sched_unit(r, blockIdx.x, gridDim.x, CAUSAL, p, u);
                if (got < 0) break;
                if (got == 0) continue;
                if (local > 0 && !mbar_wait_inl(bar_q_empty, (local - 1) & 1, abort_flag, wlim)) {
                    aborted = true;
                    break;
                }
                mbar_arrive_expect_tx(bar_q_full, 2 * TILE);
                for (int t = 0; t < 2; ++t)
                    for (int c = 0; c < C::CHUNKS; ++c)
                        tma_load_3d(&tm_q, sQ[t] + c * CHUNK_BYTES, bar_q_full, c * CHUNK_ELEMS,
                                    u.pair * UNIT_ROWS + t * BLOCK_M, u.bh);
                const int nmax = p.withhold_kv ? 0 : (u.n[0] > u.n[1] ? u.n[0] : u.n[1]);
                for (int j = 0; j < nmax; ++j) {
                    // one ring stage holds K_j and V_j, filled and released together
                    const int s = it % NSTAGE;
                    const uint32_t use = it / NSTAGE;
                    if (!mbar_wait_inl(bar_kv_empty(s), (use & 1u) ^ 1u, abort_flag, wlim)) {
                        aborted = true;
                        break;
                    }
                    mbar_arrive_expect_tx(bar_kv_full(s), 2 * TILE);
                    for (int kv = 0; kv < 2; ++kv)
                        for (int c = 0; c < C::CHUNKS; ++c) {
                            if (FP8 && kv)   // V^T: rows are d, keys run along x
                                tma_load_3d(&tm_v, sRing + (2 * s + 1) * TILE, bar_kv_full(s),
                                            j * BLOCK_N, 0, u.bh);
                            else
                                tma_load_3d(kv ? &tm_v : &tm_k,
                                            sRing + (2 * s + kv) * TILE + c * CHUNK_BYTES,
                                            bar_kv_full(s), c * CHUNK_ELEMS, j * BLOCK_N, u.bh);
                        }
                    ++it;
                }
                ++local;
                if (aborted) break;
            }
            if (aborted) {
                /* let this CTA's copies in flight land before the CTA exits */
                if (local > 0) mbar_drain_wait_inl(bar_q_full, (local - 1) & 1, wlim);
                const uint32_t n_back = it < (uint32_t)NSTAGE ? it : (uint32_t)NSTAGE;
                for (uint32_t b = 1; b <= n_back; ++b) {
                    const uint32_t i = it - b;
                    mbar_drain_wait_inl(bar_kv_full(i % NSTAGE), (i / NSTAGE) & 1u, wlim);
                }
            }
        }
        __syncwarp();
    } else if (warp == MMA_WARP) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(OTHER_REGS) : "memory");
        /* ---------------- MMA issuer ----------------
         * Tensor-core order per K/V block j (one issuing thread):
         *   P0_j V_j, S0_{j+1}, P1_j V_j, S1_{j+1}
         * so each tile's softmax of block j+1 overlaps the other tile's GEMMs.
         * S_t(j+1) overwrites the TMEM columns that hold P_t(j); the tensor
         * core runs one thread's MMAs in order, so P_t(j) V_j reads P first.
         * Waits on TMA barriers need no tcgen05 fence (no tcgen05 op precedes
         * their arrival); waits on softmax barriers do. */
        {
            // all 32 lanes run the loop (the descriptor arithmetic stays warp-uniform);
            // lane 0 issues every MMA and commit
            const uint32_t ld = lane == 0 ? 1u : 0u;
            auto wait = [&](uint32_t bar, uint32_t parity) {
                return __all_sync(0xffffffffu, mbar_wait_inl(bar, parity, abort_flag, wlim));
            };
            constexpr uint32_t IDESC_S = FP8 ? idesc_e4m3(BLOCK_M, BLOCK_N)
                                             : idesc_bf16(BLOCK_M, BLOCK_N, false);
            constexpr uint32_t IDESC_PV = FP8 ? idesc_e4m3(BLOCK_M, D) : idesc_bf16(BLOCK_M, D, true);
            constexpr uint64_t SLOT_STEP = TILE >> 4;       // descriptor units per ring slot
            const uint32_t ts0 = tmem + C::S_COL0, ts1 = tmem + C::S_COL1;
            const uint32_t to0 = tmem + C::O_COL0, to1 = tmem + C::O_COL1;
            const uint64_t qd0 = C::QK_SW64 ? sdesc_sw64(sQ[0]) : sdesc_sw128(sQ[0], 16, 1024);
            const uint64_t qd1 = C::QK_SW64 ? sdesc_sw64(sQ[1]) : sdesc_sw128(sQ[1], 16, 1024);
            const uint64_t kd_base = C::QK_SW64 ? sdesc_sw64(sRing)                   // K-major
                                                : sdesc_sw128(sRing, 16, 1024);
            const uint64_t vd_base = FP8 ? sdesc_sw128(sRing + TILE, 16, 1024)        // V^T, K-major
                                         : sdesc_sw128(sRing + TILE, CHUNK_BYTES, 1024);  // MN-major
            const uint32_t bs0 = bar_s_full0, bs1 = bar_s_full0 + 8;
            const uint32_t bh0 = bar_p_half0, bh1 = bar_p_half0 + 8;
            const uint32_t bp0 = bar_p_ready0, bp1 = bar_p_ready0 + 8;
            const uint32_t bo0 = bar_o_full0, bo1 = bar_o_full0 + 8;
            uint32_t it = 0;
            uint32_t pr0 = 0, pr1 = 0;   // p_half / p_ready phases consumed per tile
            int local = 0;
            bool aborted = false;
            for (int r = 0; !aborted; ++r) {
                Unit u;
                const int got = sched_unit(r, blockIdx.x, gridDim.x, CAUSAL, p, u);
                if (got < 0) break;
                if (got == 0) continue;
                const int n0 = u.n[0], n1 = u.n[1];
                const int nmax = n0 > n1 ? n0 : n1;
                if (!wait(bar_q_full, local & 1)) { aborted = true; break; }
                // block 0: S0_0, S1_0
                {
                    const uint32_t st = it % NSTAGE;
                    if (!wait(bar_kv_full(st), (it / NSTAGE) & 1u)) { aborted = true; break; }
                    const uint64_t kd = kd_base + 2 * st * SLOT_STEP;
                    if (n0 > 0) { issue_s<D, FP8>(ts0, qd0, kd, IDESC_S, ld); mma_commit(bs0, ld); }
                    if (n1 > 0) { issue_s<D, FP8>(ts1, qd1, kd, IDESC_S, ld); mma_commit(bs1, ld); }
                    if (nmax == 1) mma_commit(bar_q_empty, ld);
                }
                for (int j = 0; j < nmax; ++j) {
                    const uint32_t st = it % NSTAGE;                 // stage of block j
                    const uint64_t vd = vd_base + 2 * st * SLOT_STEP;
                    const uint32_t acc = j > 0 ? 1u : 0u;
                    const bool has_next = j + 1 < nmax;
                    const uint32_t nx = it + 1;                      // ring position of block j+1
                    const uint64_t kd = kd_base + 2 * (nx % NSTAGE) * SLOT_STEP;
                    if (j < n0) {
                        if (!wait(bh0, pr0 & 1u)) { aborted = true; break; }
                        tc_fence_after();
                        issue_pv<FP8>(to0, ts0, vd, IDESC_PV, acc, 0, ld);
                        if (!wait(bp0, pr0 & 1u)) { aborted = true; break; }
                        ++pr0;
                        tc_fence_after();
                        issue_pv<FP8>(to0, ts0, vd, IDESC_PV, 1u, 1, ld);
                        if (j == n0 - 1) mma_commit(bo0, ld);
                    }
                    if (has_next &&
                        !wait(bar_kv_full(nx % NSTAGE), (nx / NSTAGE) & 1u)) {
                        aborted = true;
                        break;
                    }
                    if (j + 1 < n0) { issue_s<D, FP8>(ts0, qd0, kd, IDESC_S, ld); mma_commit(bs0, ld); }
                    if (j < n1) {
                        if (!wait(bh1, pr1 & 1u)) { aborted = true; break; }
                        tc_fence_after();
                        issue_pv<FP8>(to1, ts1, vd, IDESC_PV, acc, 0, ld);
                        if (!wait(bp1, pr1 & 1u)) { aborted = true; break; }
                        ++pr1;
                        tc_fence_after();
                        issue_pv<FP8>(to1, ts1, vd, IDESC_PV, 1u, 1, ld);
                        if (j == n1 - 1) mma_commit(bo1, ld);
                    }
                    mma_commit(bar_kv_empty(st), ld);                    // K_j and V_j read
                    ++it;
                    if (j + 1 < n1) { issue_s<D, FP8>(ts1, qd1, kd, IDESC_S, ld); mma_commit(bs1, ld); }
                    if (j + 1 == nmax - 1) mma_commit(bar_q_empty, ld);  // last S of the unit issued
                }
                ++local;
            }
            /* all MMAs this thread issued have completed once this phase lands */
            mma_commit(bar_drain, ld);
            mbar_drain_wait_inl(bar_drain, 0, wlim);
        }
        __syncwarp();
    } else if (warp >= 8) {
        /* warps 10, 11: no role; their registers go to the softmax warps */
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(OTHER_REGS) : "memory");
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(SOFTMAX_REGS) : "memory");
        /* ---------------- softmax + epilogue, warps 0-7 ---------------- */
        const int t = warp >> 2;                 // Q tile of this warpgroup
        const int quarter = warp & 3;            // TMEM lanes [32*quarter, 32*quarter + 32)
        const int row_in_tile = quarter * 32 + lane;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
        const uint32_t s_addr = lane_base + (t ? C::S_COL1 : C::S_COL0);
        const uint32_t o_addr = lane_base + (t ? C::O_COL1 : C::O_COL0);
        const uint32_t bar_s = bar_s_full0 + 8 * t;
        const uint32_t bar_p = bar_p_ready0 + 8 * t;
        const uint32_t bar_ph = bar_p_half0 + 8 * t;
        const uint32_t bar_o = bar_o_full0 + 8 * t;
        const float c = p.scale_log2;
        uint32_t sph = 0, oph = 0;
        const int tail = p.N & (BLOCK_N - 1);   // valid keys in the last block (0 = full)

        for (int r = 0;; ++r) {
            Unit u;
            const int got = sched_unit(r, blockIdx.x, gridDim.x, CAUSAL, p, u);
            if (got < 0) break;
            if (got == 0) continue;
            const int n = t ? u.n[1] : u.n[0];   // (not u.n[t]: no local-memory copy of u)
            if (n == 0) continue;
            const int row = u.pair * UNIT_ROWS + t * BLOCK_M + row_in_tile;
            float m_ref = -INFINITY;   // reference max, log2 units of scale*q.k
            float l = 0.0f;            // running sum of 2^(c*s - m_ref)
            bool ok = true;
            for (int j = 0; j < n; ++j) {
                ok = mbar_wait_inl(bar_s, sph & 1u, abort_flag, wlim);
                ++sph;
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                tc_fence_after();
                uint32_t sraw[BLOCK_N];
                tmem_ld128_wait(s_addr, sraw);
                float* s = reinterpret_cast<float*>(sraw);
                if (CAUSAL && j == n - 1) {
                    // diagonal block: key column cc masked when cc > row_in_tile
#pragma unroll
                    for (int cc = 0; cc < BLOCK_N; ++cc)
                        if (cc > row_in_tile) s[cc] = -INFINITY;
                } else if (!CAUSAL && tail != 0 && j == n - 1) {
#pragma unroll
                    for (int cc = 0; cc < BLOCK_N; ++cc)
                        if (cc >= tail) s[cc] = -INFINITY;
                }
                // row max: four independent chains of three-input max
                float m8[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) m8[i] = fmaxf(s[i], s[i + 8]);
#pragma unroll
                for (int cc = 16; cc < BLOCK_N; cc += 16) {
#pragma unroll
                    for (int i = 0; i < 8; ++i) m8[i] = fmax3f(m8[i], s[cc + i], s[cc + 8 + i]);
                }
                const float mx = fmax3f(fmax3f(m8[0], m8[1], m8[2]), fmax3f(m8[3], m8[4], m8[5]),
                                        fmaxf(m8[6], m8[7]));
                const float mb = mx * c;               // block max, log2 units
                const bool need = mb > m_ref + lazy_tau<FP8>();
                float alpha = 1.0f;
                if (need) {
                    alpha = ex2(m_ref - mb);           // 0 on the first block
                    l *= alpha;
                    m_ref = mb;
                }
                // O_acc needs the factor alpha before P_j V_j lands on it.  That is
                // rare with lazy rescaling, so a warp that needs it stores all of
                // P first (the scores are dead by then) and hands P over after
                // the rescale; otherwise P goes over in two halves so the first
                // half of P V starts while the second half is computed.
                const bool warp_rescale = j > 0 && __any_sync(0xffffffffu, need);
                const float neg_m = (m_ref == -INFINITY) ? 0.0f : -m_ref;
                const uint64_t c2 = f2pack(c, c);
                const uint64_t nm2 = f2pack(neg_m, neg_m);
                uint64_t sum2 = f2pack(0.0f, 0.0f);
#pragma unroll
                for (int qtr = 0; qtr < 4; ++qtr) {
                    const int half = qtr >> 1;
                    uint32_t pk[BLOCK_N / 8];
                    float pq[FP8 ? BLOCK_N / 4 : 1];
#pragma unroll
                    for (int k = 0; k < BLOCK_N / 8; ++k) {
                        const int cc = qtr * (BLOCK_N / 4) + 2 * k;
                        float x0, x1;
                        f2unpack(ffma2(f2pack(s[cc], s[cc + 1]), c2, nm2), x0, x1);
                        float p0, p1;
                        if ((exp2_poly_mask<D, FP8>() >> ((qtr * (BLOCK_N / 8) + k) & 7)) & 1u) {
                            exp2_poly_pair(x0, x1, p0, p1);
                        } else {
                            p0 = ex2(x0);
                            p1 = ex2(x1);
                        }
                        sum2 = fadd2(sum2, f2pack(p0, p1));
                        if constexpr (FP8) {
                            pq[2 * k] = p0;
                            pq[2 * k + 1] = p1;
                        } else {
                            pk[k] = pack_bf16(p0, p1);
                        }
                    }
                    if constexpr (FP8) {
                        uint32_t p8[BLOCK_N / 16];
#pragma unroll
                        for (int e = 0; e < BLOCK_N / 16; ++e)
                            p8[e] = pack_e4m3x4(pq[4 * e], pq[4 * e + 1], pq[4 * e + 2], pq[4 * e + 3]);
                        tmem_st8(s_addr + qtr * (BLOCK_N / 16), p8);
                    } else {
                        tmem_st16(s_addr + qtr * (BLOCK_N / 8), pk);
                    }
                    if (!warp_rescale && (qtr & 1)) {
                        tmem_wait_st();
                        tc_fence_before();
                        mbar_arrive(half ? bar_p : bar_ph);
                    }
                }
                if (warp_rescale) {
                    // PV of block j-1 has completed: the commit that released S_j
                    // covers it, so O_acc is stable here
#pragma unroll
                    for (int ch = 0; ch < D / 32; ++ch) {
                        uint32_t ov[32];
                        tmem_ld32_wait(o_addr + ch * 32, ov);
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
                        tmem_st32(o_addr + ch * 32, ov);
                    }
                    tmem_wait_st();
                    tc_fence_before();
                    mbar_arrive(bar_ph);
                    mbar_arrive(bar_p);
                }
                {
                    float sa, sb;
                    f2unpack(sum2, sa, sb);
                    l += sa + sb;
                }
            }
            if (!ok) break;
            ok = mbar_wait_inl(bar_o, oph & 1u, abort_flag, wlim);
            ++oph;
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            float inv_l = l > 0.0f ? 1.0f / l : 0.0f;
            if constexpr (FP8) inv_l *= p.o_scale;
            const bool live = row < p.N;
            __nv_bfloat16* orow = p.o + (static_cast<size_t>(u.bh) * p.N + (live ? row : 0)) * D;
#pragma unroll
            for (int ch = 0; ch < D / 32; ++ch) {
                uint32_t ov[32];
                tmem_ld32_wait(o_addr + ch * 32, ov);
                uint32_t w[16];
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    w[e] = pack_bf16(__uint_as_float(ov[2 * e]) * inv_l,
                                     __uint_as_float(ov[2 * e + 1]) * inv_l);
                if (live) {
                    uint4* dst = reinterpret_cast<uint4*>(orow + ch * 32);
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        dst[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
                }
            }
            if (live) p.lse[static_cast<size_t>(u.bh) * p.N + row] = (m_ref + log2f(l)) * LN2;
            tc_fence_before();
        }
    }

    /* ---------------- teardown ---------------- */
    tc_fence_before();
    __syncthreads();
    if (warp == MMA_WARP) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS)
                     : "memory");
    }
}

}  // namespace
/* ------------------------------------------------------------------------ */
/* Host side: validation, tensor maps, launch                                */
/* ------------------------------------------------------------------------ */
namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

constexpr int MAX_DEVICES = 64;

/* Per-device state.  What depends on the CUDA context (kernel attributes set
 * with cudaFuncSetAttribute, the device address of a __device__ symbol) is
 * keyed by the id of the context current on the calling thread: after a
 * cudaDeviceReset, or with another context made current, it is set up again
 * instead of being reused. */
struct DeviceInfo {
    bool ready = false;
    int status = ATTN_OK;   // ATTN_ERR_DEVICE when the device is not CC 10.0
    int num_sms = 0;
    unsigned long long ctx_id = 0;   // context the flags and addresses below belong to
    bool ctx_known = false;
    bool smem_set[8] = {};           // forward kernels: (FP8, D == 128, CAUSAL)
    bool bwd_set[4] = {};            // backward kernels: (D == 128, CAUSAL)
    bool dec_set[2] = {};            // decode stream kernels: D == 128
    bool std_set[2] = {};            // standard-path GEMM kernels: D == 128
    void* scratch = nullptr;         // device address of the no-alloc decode buffer
    bool host_ready = false;         // helper streams and events of attn_fwd_host below
    cudaStream_t host_streams[3] = {};   // copies in, kernels, copies out
    cudaEvent_t host_events[4] = {};     // start, chunk copied in, chunk computed, done
};

std::mutex g_mutex;
DeviceInfo g_dev[MAX_DEVICES];
EncodeTiledFn g_encode = nullptr;

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);
CtxGetCurrentFn g_ctx_current = nullptr;
CtxGetIdFn g_ctx_get_id = nullptr;

/* A driver entry point by name (the library links the runtime only). */
bool driver_entry(const char* name, void** fn) {
    cudaDriverEntryPointQueryResult qres;
    if (cudaGetDriverEntryPoint(name, fn, cudaEnableDefault, &qres) != cudaSuccess ||
        qres != cudaDriverEntryPointSuccess || !*fn) {
        cudaGetLastError();
        return false;
    }
    return true;
}

int get_encode(EncodeTiledFn* fn) {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_encode) {
        void* ptr = nullptr;
        if (!driver_entry("cuTensorMapEncodeTiled", &ptr)) return ATTN_ERR_CUDA;
        g_encode = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    *fn = g_encode;
    return ATTN_OK;
}

/* Process-unique id of the context current on this thread (caller holds
 * g_mutex).  If none is current yet, a symbol lookup makes the runtime bind
 * its primary context first. */
int current_context_id(unsigned long long* id) {
    if (!g_ctx_current || !g_ctx_get_id) {
        void* a = nullptr;
        void* b = nullptr;
        if (!driver_entry("cuCtxGetCurrent", &a) || !driver_entry("cuCtxGetId", &b))
            return ATTN_ERR_CUDA;
        g_ctx_current = reinterpret_cast<CtxGetCurrentFn>(a);
        g_ctx_get_id = reinterpret_cast<CtxGetIdFn>(b);
    }
    CUcontext ctx = nullptr;
    if (g_ctx_current(&ctx) != CUDA_SUCCESS) return ATTN_ERR_CUDA;
    if (!ctx) {
        void* sym = nullptr;
        if (cudaGetSymbolAddress(&sym, g_attn_status) != cudaSuccess) {
            cudaGetLastError();
            return ATTN_ERR_CUDA;
        }
        if (g_ctx_current(&ctx) != CUDA_SUCCESS || !ctx) return ATTN_ERR_CUDA;
    }
    return g_ctx_get_id(ctx, id) == CUDA_SUCCESS ? ATTN_OK : ATTN_ERR_CUDA;
}

int device_info(int* dev_out, DeviceInfo** info_out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) { cudaGetLastError(); return ATTN_ERR_CUDA; }
    if (dev < 0 || dev >= MAX_DEVICES) return ATTN_ERR_DEVICE;
    std::lock_guard<std::mutex> lock(g_mutex);
    DeviceInfo& di = g_dev[dev];
    if (!di.ready) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
            cudaGetLastError();
            return ATTN_ERR_CUDA;
        }
        di.status = (major == 10 && minor == 0) ? ATTN_OK : ATTN_ERR_DEVICE;
        di.num_sms = sms;
        di.ready = true;
    }
    if (di.status != ATTN_OK) return di.status;
    unsigned long long id = 0;
    const int st = current_context_id(&id);
    if (st != ATTN_OK) return st;
    if (!di.ctx_known || di.ctx_id != id) {   // first call in this context: set up again
        for (int i = 0; i < 8; ++i) di.smem_set[i] = false;
        for (int i = 0; i < 4; ++i) di.bwd_set[i] = false;
        for (int i = 0; i < 2; ++i) di.dec_set[i] = di.std_set[i] = false;
        di.scratch = nullptr;
        di.host_ready = false;   // streams and events of another context are not used here
        di.ctx_id = id;
        di.ctx_known = true;
    }
    *dev_out = dev;
    *info_out = &di;
    return ATTN_OK;
}

/* 3-D view [B*H][N][d] of a bf16 tensor, box = 64 columns x 128 rows x 1 head,
 * 128-byte swizzle; rows past N read as zeros. */
int encode_map(EncodeTiledFn fn, CUtensorMap* map, const void* ptr, int64_t BH, int64_t N,
               int64_t d, uint32_t box_rows = BLOCK_M) {
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                          static_cast<cuuint64_t>(BH)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(d * 2), static_cast<cuuint64_t>(N * d * 2)};
    cuuint32_t box[3] = {CHUNK_ELEMS, box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? ATTN_OK : ATTN_ERR_CUDA;
}

bool ranges_overlap(const void* a, size_t na, const void* b, size_t nb) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

/* Argument checks shared by the device and host entry points (no CUDA calls). */
int validate_shape(int64_t B, int64_t H, int64_t N, int64_t d, float scale, bool* empty) {
    if (B < 0 || H < 0 || N < 0) return ATTN_ERR_SHAPE;
    if (d != 64 && d != 128) return ATTN_ERR_HEADDIM;
    if (!(scale > 0.0f) || !isfinite(scale)) return ATTN_ERR_SCALE;
    *empty = (B == 0 || H == 0 || N == 0);
    if (*empty) return ATTN_OK;
    if (N > INT32_MAX - 2 * UNIT_ROWS) return ATTN_ERR_SHAPE;
    if (H > INT32_MAX / B) return ATTN_ERR_SHAPE;
    const int64_t BH = B * H;
    const int64_t n_pairs = (N + UNIT_ROWS - 1) / UNIT_ROWS;
    if (BH > INT32_MAX / n_pairs) return ATTN_ERR_SHAPE;   // unit index fits int32
    return ATTN_OK;
}

template <int D, bool CAUSAL, bool FP8 = false>
int launch(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
           const FwdParams& prm, DeviceInfo* di, cudaStream_t stream) {
    auto kern = attn_fwd_sm100_kernel<D, CAUSAL, FP8>;
    constexpr int SMEM = Cfg<D, FP8>::SMEM_BYTES;
    const int key = (FP8 ? 4 : 0) + (D == 128 ? 2 : 0) + (CAUSAL ? 1 : 0);
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        if (!di->smem_set[key]) {
            // the register split adds up only with LAUNCH_REGS per thread: with
            // fewer, setmaxnreg.inc would wait for registers that never come free
            cudaFuncAttributes fa;
            if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess || fa.numRegs != LAUNCH_REGS ||
                cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM) !=
                    cudaSuccess) {
                cudaGetLastError();
                return ATTN_ERR_LAUNCH;
            }
            di->smem_set[key] = true;
        }
    }
    const int grid = prm.n_units < di->num_sms ? prm.n_units : di->num_sms;
    FwdParams sp = prm;
    plan_schedule(sp, grid);
    kern<<<grid, NUM_THREADS, SMEM, stream>>>(mq, mk, mv, sp);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_LAUNCH;
    return ATTN_OK;
}

/* The forward call behind attn_fwd and the timeout test hook. */
int fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B,
             int64_t H, int64_t N, int64_t d, int causal, float scale, void* stream,
             uint64_t wait_limit_ns, int withhold_kv) {
    bool empty = false;
    int st = validate_shape(B, H, N, d, scale, &empty);
    if (st != ATTN_OK || empty) return st;
    if (!q || !k || !v || !o || !lse) return ATTN_ERR_NULL;
    const void* ptrs[5] = {q, k, v, o, lse};
    for (const void* ptr : ptrs)
        if (reinterpret_cast<uintptr_t>(ptr) & 15u) return ATTN_ERR_ALIGN;
    const size_t tbytes = static_cast<size_t>(B * H * N * d) * 2;
    const size_t lbytes = static_cast<size_t>(B * H * N) * 4;
    if (ranges_overlap(o, tbytes, q, tbytes) || ranges_overlap(o, tbytes, k, tbytes) ||
        ranges_overlap(o, tbytes, v, tbytes) || ranges_overlap(lse, lbytes, q, tbytes) ||
        ranges_overlap(lse, lbytes, k, tbytes) || ranges_overlap(lse, lbytes, v, tbytes) ||
        ranges_overlap(lse, lbytes, o, tbytes))
        return ATTN_ERR_OVERLAP;

    int dev = 0;
    DeviceInfo* di = nullptr;
    if ((st = device_info(&dev, &di)) != ATTN_OK) return st;
    EncodeTiledFn enc = nullptr;
    if ((st = get_encode(&enc)) != ATTN_OK) return st;
    const int64_t BH = B * H;
    CUtensorMap mq, mk, mv;
    if ((st = encode_map(enc, &mq, q, BH, N, d)) != ATTN_OK) return st;
    if ((st = encode_map(enc, &mk, k, BH, N, d)) != ATTN_OK) return st;
    if ((st = encode_map(enc, &mv, v, BH, N, d)) != ATTN_OK) return st;

    FwdParams prm;
    prm.o = static_cast<__nv_bfloat16*>(o);
    prm.lse = lse;
    prm.N = static_cast<int>(N);
    prm.BH = static_cast<int>(BH);
    prm.n_pairs = static_cast<int>((N + UNIT_ROWS - 1) / UNIT_ROWS);
    prm.nkv = static_cast<int>((N + BLOCK_N - 1) / BLOCK_N);
    prm.n_units = prm.BH * prm.n_pairs;
    prm.scale_log2 = scale * LOG2E;
    prm.wait_limit_ns = wait_limit_ns;
    prm.withhold_kv = withhold_kv;
    prm.o_scale = 1.0f;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (d == 64)
        return causal ? launch<64, true>(mq, mk, mv, prm, di, s) : launch<64, false>(mq, mk, mv, prm, di, s);
    return causal ? launch<128, true>(mq, mk, mv, prm, di, s) : launch<128, false>(mq, mk, mv, prm, di, s);
}

/* ------------------------------------------------------------------------ */
/* e4m3 inputs: V transposed into the workspace, then the same kernel        */
/* ------------------------------------------------------------------------ */
/* V [BH, N, D] e4m3 -> V^T [BH, D, Np] (Np = N rounded up to 128; keys past N
 * are zero, so masked keys multiply zeros).  One CTA of 2 D threads per (head,
 * block of 128 keys).  A thread reads four keys x 16 bytes, transposes the
 * 4 x 4 byte blocks in registers and parks 32-bit words (4 keys of one column)
 * in shared memory; the CTA then writes the block's D rows of V^T with 16-byte
 * stores. */
__device__ __forceinline__ void transpose4x4_bytes(const uint32_t w[4], uint32_t out[4]) {
    // out[c] = byte c of w[0], w[1], w[2], w[3] (w[r] in byte r)
    const uint32_t lo01 = __byte_perm(w[0], w[1], 0x5140), hi01 = __byte_perm(w[0], w[1], 0x7362);
    const uint32_t lo23 = __byte_perm(w[2], w[3], 0x5140), hi23 = __byte_perm(w[2], w[3], 0x7362);
    out[0] = __byte_perm(lo01, lo23, 0x5410);
    out[1] = __byte_perm(lo01, lo23, 0x7632);
    out[2] = __byte_perm(hi01, hi23, 0x5410);
    out[3] = __byte_perm(hi01, hi23, 0x7632);
}

template <int D>
__global__ void __launch_bounds__(2 * D)
fp8_transpose_v_kernel(const uint8_t* __restrict__ v, uint8_t* __restrict__ vt, int N, int Np) {
    constexpr int C16 = D / 16;               // 16-byte pieces of a V row
    __shared__ uint32_t tw[D][33];            // [column][group of 4 keys], padded row
    const int kb = blockIdx.x, bh = blockIdx.y, t = threadIdx.x;
    const uint8_t* src = v + (static_cast<int64_t>(bh) * N + static_cast<int64_t>(kb) * 128) * D;
    {
        const int g = t / C16, c16 = t % C16;  // keys 4g .. 4g+3, columns 16 c16 .. 16 c16 + 15
        uint4 rows[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int key = 4 * g + r;
            rows[r] = make_uint4(0u, 0u, 0u, 0u);
            if (kb * 128 + key < N)
                rows[r] = *reinterpret_cast<const uint4*>(src + key * D + c16 * 16);
        }
#pragma unroll
        for (int wi = 0; wi < 4; ++wi) {
            const uint32_t w[4] = {wi == 0 ? rows[0].x : wi == 1 ? rows[0].y : wi == 2 ? rows[0].z : rows[0].w,
                                   wi == 0 ? rows[1].x : wi == 1 ? rows[1].y : wi == 2 ? rows[1].z : rows[1].w,
                                   wi == 0 ? rows[2].x : wi == 1 ? rows[2].y : wi == 2 ? rows[2].z : rows[2].w,
                                   wi == 0 ? rows[3].x : wi == 1 ? rows[3].y : wi == 2 ? rows[3].z : rows[3].w};
            uint32_t out[4];
            transpose4x4_bytes(w, out);
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) tw[c16 * 16 + wi * 4 + cc][g] = out[cc];
        }
    }
    __syncthreads();
    uint8_t* dst = vt + static_cast<int64_t>(bh) * D * Np + static_cast<int64_t>(kb) * 128;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int item = t + 2 * D * i;       // D columns x 8 runs of 16 keys
        const int col = item >> 3, u = item & 7;
        *reinterpret_cast<uint4*>(dst + static_cast<int64_t>(col) * Np + u * 16) =
            make_uint4(tw[col][4 * u], tw[col][4 * u + 1], tw[col][4 * u + 2], tw[col][4 * u + 3]);
    }
}

/* 3-D map over 8-bit data [BH][rows][inner], box box_inner bytes x box_rows
 * rows: 128-byte swizzle for 128-byte box rows, 64-byte swizzle for 64-byte ones. */
int encode_map_u8(EncodeTiledFn fn, CUtensorMap* map, const void* ptr, int64_t BH, int64_t rows,
                  int64_t inner, uint32_t box_inner = 128, uint32_t box_rows = BLOCK_M) {
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(rows),
                          static_cast<cuuint64_t>(BH)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(rows * inner)};
    cuuint32_t box[3] = {box_inner, box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    box_inner == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? ATTN_OK : ATTN_ERR_CUDA;
}

size_t fp8_ws_bytes(int64_t BH, int64_t N, int64_t d) {
    const int64_t Np = (N + BLOCK_N - 1) / BLOCK_N * BLOCK_N;
    return static_cast<size_t>(BH) * d * Np;
}

int fp8_impl(const void* q, const void* k, const void* v, float q_descale, float k_descale,
             float v_descale, void* o, float* lse, int64_t B, int64_t H, int64_t N, int64_t d,
             int causal, float scale, void* workspace, size_t workspace_bytes, void* stream) {
    bool empty = false;
    int st = validate_shape(B, H, N, d, scale, &empty);
    if (st != ATTN_OK) return st;
    if (empty) return ATTN_OK;
    if (B * H > 65535) return ATTN_ERR_SHAPE;
    const float ds[3] = {q_descale, k_descale, v_descale};
    for (float x : ds)
        if (!(x > 0.0f) || !isfinite(x)) return ATTN_ERR_SCALE;
    if (!isfinite(scale * q_descale * k_descale * LOG2E)) return ATTN_ERR_SCALE;
    const void* ptrs[5] = {q, k, v, o, lse};
    for (const void* ptr : ptrs) {
        if (!ptr) return ATTN_ERR_NULL;
        if (reinterpret_cast<uintptr_t>(ptr) & 15u) return ATTN_ERR_ALIGN;
    }
    const int64_t BH = B * H;
    const size_t ws_need = fp8_ws_bytes(BH, N, d);
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < ws_need)
        return ATTN_ERR_WORKSPACE;
    const size_t in_bytes = static_cast<size_t>(BH * N * d);
    const size_t obytes = in_bytes * 2, lbytes = static_cast<size_t>(BH * N) * 4;
    const void* ins[3] = {q, k, v};
    for (const void* in : ins)
        if (ranges_overlap(o, obytes, in, in_bytes) || ranges_overlap(lse, lbytes, in, in_bytes) ||
            ranges_overlap(workspace, ws_need, in, in_bytes))
            return ATTN_ERR_OVERLAP;
    if (ranges_overlap(o, obytes, lse, lbytes) || ranges_overlap(workspace, ws_need, o, obytes) ||
        ranges_overlap(workspace, ws_need, lse, lbytes))
        return ATTN_ERR_OVERLAP;
    int dev = 0;
    DeviceInfo* di = nullptr;
    if ((st = device_info(&dev, &di)) != ATTN_OK) return st;
    EncodeTiledFn enc = nullptr;
    if ((st = get_encode(&enc)) != ATTN_OK) return st;
    const int64_t Np = (N + BLOCK_N - 1) / BLOCK_N * BLOCK_N;
    CUtensorMap mq, mk, mvt;
    const uint32_t qk_box = static_cast<uint32_t>(d);   // a Q / K row: 128 or 64 bytes
    if ((st = encode_map_u8(enc, &mq, q, BH, N, d, qk_box)) != ATTN_OK) return st;
    if ((st = encode_map_u8(enc, &mk, k, BH, N, d, qk_box)) != ATTN_OK) return st;
    if ((st = encode_map_u8(enc, &mvt, workspace, BH, d, Np, 128, static_cast<uint32_t>(d))) != ATTN_OK)
        return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const dim3 tgrid(static_cast<unsigned>(Np / BLOCK_N), static_cast<unsigned>(BH));
    if (d == 64)
        fp8_transpose_v_kernel<64><<<tgrid, 128, 0, s>>>(static_cast<const uint8_t*>(v),
                                                         static_cast<uint8_t*>(workspace),
                                                         static_cast<int>(N), static_cast<int>(Np));
    else
        fp8_transpose_v_kernel<128><<<tgrid, 256, 0, s>>>(static_cast<const uint8_t*>(v),
                                                          static_cast<uint8_t*>(workspace),
                                                          static_cast<int>(N), static_cast<int>(Np));
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_LAUNCH;
    FwdParams prm;
    prm.o = static_cast<__nv_bfloat16*>(o);
    prm.lse = lse;
    prm.N = static_cast<int>(N);
    prm.BH = static_cast<int>(BH);
    prm.n_pairs = static_cast<int>((N + UNIT_ROWS - 1) / UNIT_ROWS);
    prm.nkv = static_cast<int>(Np / BLOCK_N);
    prm.n_units = prm.BH * prm.n_pairs;
    prm.scale_log2 = scale * q_descale * k_descale * LOG2E;
    prm.wait_limit_ns = WAIT_LIMIT_NS;
    prm.withhold_kv = 0;
    prm.o_scale = v_descale;
    if (d == 64)
        return causal ? launch<64, true, true>(mq, mk, mvt, prm, di, s)
                      : launch<64, false, true>(mq, mk, mvt, prm, di, s);
    return causal ? launch<128, true, true>(mq, mk, mvt, prm, di, s)
                  : launch<128, false, true>(mq, mk, mvt, prm, di, s);
}

/* Everything above is the forward pass; the standard path and the backward
 * pass follow. */
#include "attn_standard.cuh"

/* ATTN_ERR_OVERLAP when an output range (a device workspace counts as one)
 * overlaps an input range or another output range; checked before any launch. */
int check_overlaps(const void* const* outs, const size_t* out_bytes, int n_out,
                   const void* const* ins, const size_t* in_bytes, int n_in) {
    for (int a = 0; a < n_out; ++a) {
        for (int b = 0; b < n_in; ++b)
            if (ranges_overlap(outs[a], out_bytes[a], ins[b], in_bytes[b])) return ATTN_ERR_OVERLAP;
        for (int b = a + 1; b < n_out; ++b)
            if (ranges_overlap(outs[a], out_bytes[a], outs[b], out_bytes[b])) return ATTN_ERR_OVERLAP;
    }
    return ATTN_OK;
}

/* The unfused three-kernel path (S and P through device memory), host side. */
size_t std_ws_bytes(int64_t BH, int64_t N) {
    const int64_t Np = (N + BLOCK_M - 1) / BLOCK_M * BLOCK_M;
    return static_cast<size_t>(BH) * Np * Np * sizeof(float);
}

int std_validate(int64_t B, int64_t H, int64_t N, int64_t d, float scale, bool* empty) {
    int st = validate_shape(B, H, N, d, scale, empty);
    if (st != ATTN_OK || *empty) return st;
    if (N > STD_MAX_N || B * H > 65535) return ATTN_ERR_SHAPE;
    return ATTN_OK;
}

template <int D>
int std_launch(const void* q, const void* k, const void* v, const StdParams& prm,
               EncodeTiledFn enc, DeviceInfo* di, cudaStream_t stream) {
    CUtensorMap mq, mk, mv, mp;
    int st;
    if ((st = encode_map(enc, &mq, q, prm.BH, prm.N, D)) != ATTN_OK) return st;
    if ((st = encode_map(enc, &mk, k, prm.BH, prm.N, D)) != ATTN_OK) return st;
    if ((st = encode_map(enc, &mv, v, prm.BH, prm.N, D, STD_PV_KEYS)) != ATTN_OK) return st;
    {   // P: bf16 over the first half of every fp32 S row (row pitch 4 * Np bytes)
        const int64_t Np = prm.Np;
        cuuint64_t dims[3] = {static_cast<cuuint64_t>(Np), static_cast<cuuint64_t>(Np),
                              static_cast<cuuint64_t>(prm.BH)};
        cuuint64_t strides[2] = {static_cast<cuuint64_t>(Np * 4),
                                 static_cast<cuuint64_t>(Np * Np * 4)};
        cuuint32_t box[3] = {STD_PV_KEYS, BLOCK_M, 1};
        cuuint32_t estr[3] = {1, 1, 1};
        if (enc(&mp, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, prm.S, dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) !=
            CUDA_SUCCESS)
            return ATTN_ERR_CUDA;
    }
    // kernel 1 keeps at most 3-4 CTAs per SM so their TMEM columns fit
    const int smem1 = (2 * BLOCK_M * D * 2 > 56 * 1024 ? 2 * BLOCK_M * D * 2 : 56 * 1024) + 2048;
    constexpr int stage = BLOCK_M * STD_PV_KEYS * 2 + STD_PV_KEYS * D * 2;
    const int smem3 = STD_PV_STAGES * stage + 16 * STD_PV_STAGES + 64 + 1024;
    auto k1 = std_qk_kernel<D>;
    auto k3 = std_pv_kernel<D>;
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        bool& set = di->std_set[D == 128 ? 1 : 0];
        if (!set) {
            if (cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, smem1) !=
                    cudaSuccess ||
                cudaFuncSetAttribute(k3, cudaFuncAttributeMaxDynamicSharedMemorySize, smem3) !=
                    cudaSuccess) {
                cudaGetLastError();
                return ATTN_ERR_LAUNCH;
            }
            set = true;
        }
    }
    const unsigned tiles = static_cast<unsigned>(prm.Np / BLOCK_M);
    k1<<<dim3(tiles, tiles, prm.BH), STD_THREADS, smem1, stream>>>(mq, mk, prm);
    const int64_t rows = static_cast<int64_t>(prm.BH) * prm.N;
    if (prm.Np <= STD_SHORT_MAX_NP) {
        const int64_t per = STD_SOFTMAX_THREADS / 32;
        std_softmax_short_kernel<<<static_cast<unsigned>((rows + per - 1) / per),
                                   STD_SOFTMAX_THREADS, 0, stream>>>(prm);
    } else {
        const unsigned g = static_cast<unsigned>(rows);
        if (prm.Np <= 4 * STD_SOFTMAX_THREADS * 4)
            std_softmax_kernel<4><<<g, STD_SOFTMAX_THREADS, 0, stream>>>(prm);
        else if (prm.Np <= 4 * STD_SOFTMAX_THREADS * 8)
            std_softmax_kernel<8><<<g, STD_SOFTMAX_THREADS, 0, stream>>>(prm);
        else if (prm.Np <= 4 * STD_SOFTMAX_THREADS * 16)
            std_softmax_kernel<16><<<g, STD_SOFTMAX_THREADS, 0, stream>>>(prm);
        else
            std_softmax_kernel<STD_MAX_N / (4 * STD_SOFTMAX_THREADS)><<<g, STD_SOFTMAX_THREADS, 0, stream>>>(prm);
    }
    k3<<<dim3(tiles, prm.BH), STD_THREADS, smem3, stream>>>(mp, mv, prm);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_LAUNCH;
    return ATTN_OK;
}

int std_impl(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B,
             int64_t H, int64_t N, int64_t d, int causal, float scale, void* workspace,
             size_t workspace_bytes, void* stream) {
    bool empty = false;
    int st = std_validate(B, H, N, d, scale, &empty);
    if (st != ATTN_OK || empty) return st;
    if (!q || !k || !v || !o || !lse) return ATTN_ERR_NULL;
    const void* ptrs[5] = {q, k, v, o, lse};
    for (const void* ptr : ptrs)
        if (reinterpret_cast<uintptr_t>(ptr) & 15u) return ATTN_ERR_ALIGN;
    const int64_t BH = B * H;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
        workspace_bytes < std_ws_bytes(BH, N))
        return ATTN_ERR_WORKSPACE;
    {
        const size_t tb = static_cast<size_t>(BH * N * d) * 2, lb = static_cast<size_t>(BH * N) * 4;
        const void* outs[3] = {o, lse, workspace};
        const size_t ob[3] = {tb, lb, std_ws_bytes(BH, N)};
        const void* ins[3] = {q, k, v};
        const size_t ib[3] = {tb, tb, tb};
        if ((st = check_overlaps(outs, ob, 3, ins, ib, 3)) != ATTN_OK) return st;
    }
    int dev = 0;
    DeviceInfo* di = nullptr;
    if ((st = device_info(&dev, &di)) != ATTN_OK) return st;
    EncodeTiledFn enc = nullptr;
    if ((st = get_encode(&enc)) != ATTN_OK) return st;
    StdParams prm;
    prm.S = static_cast<float*>(workspace);
    prm.lse = lse;
    prm.o = static_cast<__nv_bfloat16*>(o);
    prm.N = static_cast<int>(N);
    prm.Np = static_cast<int>((N + BLOCK_M - 1) / BLOCK_M * BLOCK_M);
    prm.BH = static_cast<int>(BH);
    prm.causal = causal ? 1 : 0;
    prm.scale = scale;
    prm.wait_limit_ns = WAIT_LIMIT_NS;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    return d == 64 ? std_launch<64>(q, k, v, prm, enc, di, s) : std_launch<128>(q, k, v, prm, enc, di, s);
}

#include "attn_bwd.cuh"

/* Backward pass, host side.  Workspace: the tiled dQ accumulator (fp32,
 * BH * Np * d values), D and LSE*log2(e) (fp32 [BH, Np] each), 256-byte
 * aligned pieces. */
size_t bwd_ws_bytes(int64_t BH, int64_t N, int64_t d) {
    const int64_t Np = (N + BLOCK_M - 1) / BLOCK_M * BLOCK_M;
    auto a256 = [](size_t x) { return (x + 255u) & ~static_cast<size_t>(255u); };
    return a256(static_cast<size_t>(BH) * Np * d * 4) + 2 * a256(static_cast<size_t>(BH) * Np * 4);
}

template <int D, bool CAUSAL>
int bwd_launch(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
               const CUtensorMap& mdo, const __nv_bfloat16* o, const __nv_bfloat16* dout,
               const float* lse, const BwdParams& prm, DeviceInfo* di, cudaStream_t stream) {
    auto kern = bwd_main_kernel<D, CAUSAL>;
    constexpr int SMEM = BwdCfg<D>::SMEM_BYTES;
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        bool& set = di->bwd_set[(D == 128 ? 2 : 0) + (CAUSAL ? 1 : 0)];
        if (!set) {
            // the register split adds up only with BWD_LAUNCH_REGS per thread (see attn_bwd.cuh)
            cudaFuncAttributes fa;
            if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess || fa.numRegs != BWD_LAUNCH_REGS ||
                cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM) !=
                    cudaSuccess) {
                cudaGetLastError();
                return ATTN_ERR_LAUNCH;
            }
            set = true;
        }
    }
    const int64_t prows = static_cast<int64_t>(prm.BH) * prm.Np;
    if (cudaMemsetAsync(prm.dq_acc, 0, static_cast<size_t>(prows) * D * 4, stream) != cudaSuccess)
        return ATTN_ERR_CUDA;
    constexpr int pre_rows = BWD_PRE_THREADS / (D / 8);
    bwd_pre_kernel<D><<<static_cast<unsigned>((prows + pre_rows - 1) / pre_rows), BWD_PRE_THREADS, 0,
                        stream>>>(
        o, dout, lse, const_cast<float*>(prm.Dp), const_cast<float*>(prm.lse2), prm.N, prm.Np,
        prm.BH);
    kern<<<static_cast<unsigned>(prm.nblk * prm.BH), BWD_THREADS, SMEM, stream>>>(mq, mk, mv, mdo, prm);
    bwd_post_kernel<D><<<static_cast<unsigned>(prm.BH * prm.nblk), BLOCK_M, 0, stream>>>(
        prm.dq_acc, prm.dq, prm.N, prm.nblk);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_LAUNCH;
    return ATTN_OK;
}

int bwd_impl(const void* q, const void* k, const void* v, const void* o, const void* dout,
             const float* lse, void* dq, void* dk, void* dv, int64_t B, int64_t H, int64_t N,
             int64_t d, int causal, float scale, void* workspace, size_t workspace_bytes,
             void* stream, uint64_t wait_limit_ns, int withhold) {
    bool empty = false;
    int st = validate_shape(B, H, N, d, scale, &empty);
    if (st != ATTN_OK || empty) return st;
    if (B * H > 65535) return ATTN_ERR_SHAPE;
    const void* ptrs[9] = {q, k, v, o, dout, lse, dq, dk, dv};
    for (const void* ptr : ptrs) {
        if (!ptr) return ATTN_ERR_NULL;
        if (reinterpret_cast<uintptr_t>(ptr) & 15u) return ATTN_ERR_ALIGN;
    }
    const int64_t BH = B * H;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
        workspace_bytes < bwd_ws_bytes(BH, N, d))
        return ATTN_ERR_WORKSPACE;
    {
        const size_t tb = static_cast<size_t>(BH * N * d) * 2, lb = static_cast<size_t>(BH * N) * 4;
        const void* outs[4] = {dq, dk, dv, workspace};
        const size_t ob[4] = {tb, tb, tb, bwd_ws_bytes(BH, N, d)};
        const void* ins[6] = {q, k, v, o, dout, lse};
        const size_t ib[6] = {tb, tb, tb, tb, tb, lb};
        if ((st = check_overlaps(outs, ob, 4, ins, ib, 6)) != ATTN_OK) return st;
    }
    int dev = 0;
    DeviceInfo* di = nullptr;
    if ((st = device_info(&dev, &di)) != ATTN_OK) return st;
    EncodeTiledFn enc = nullptr;
    if ((st = get_encode(&enc)) != ATTN_OK) return st;
    CUtensorMap mq, mk, mv, mdo;
    if ((st = encode_map(enc, &mq, q, BH, N, d)) != ATTN_OK) return st;
    if ((st = encode_map(enc, &mk, k, BH, N, d)) != ATTN_OK) return st;
    if ((st = encode_map(enc, &mv, v, BH, N, d)) != ATTN_OK) return st;
    if ((st = encode_map(enc, &mdo, dout, BH, N, d)) != ATTN_OK) return st;
    const int64_t Np = (N + BLOCK_M - 1) / BLOCK_M * BLOCK_M;
    auto a256 = [](size_t x) { return (x + 255u) & ~static_cast<size_t>(255u); };
    char* ws = static_cast<char*>(workspace);
    BwdParams prm;
    prm.dq = static_cast<__nv_bfloat16*>(dq);
    prm.dk = static_cast<__nv_bfloat16*>(dk);
    prm.dv = static_cast<__nv_bfloat16*>(dv);
    prm.dq_acc = reinterpret_cast<float*>(ws);
    prm.Dp = reinterpret_cast<float*>(ws + a256(static_cast<size_t>(BH) * Np * d * 4));
    prm.lse2 = prm.Dp + (a256(static_cast<size_t>(BH) * Np * 4) / 4);
    prm.N = static_cast<int>(N);
    prm.Np = static_cast<int>(Np);
    prm.BH = static_cast<int>(BH);
    prm.nblk = static_cast<int>(Np / BLOCK_M);
    prm.scale = scale;
    prm.scale_log2 = scale * LOG2E;
    prm.wait_limit_ns = wait_limit_ns;
    prm.withhold = withhold;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const auto* ob = static_cast<const __nv_bfloat16*>(o);
    const auto* db = static_cast<const __nv_bfloat16*>(dout);
    if (d == 64)
        return causal ? bwd_launch<64, true>(mq, mk, mv, mdo, ob, db, lse, prm, di, s)
                      : bwd_launch<64, false>(mq, mk, mv, mdo, ob, db, lse, prm, di, s);
    return causal ? bwd_launch<128, true>(mq, mk, mv, mdo, ob, db, lse, prm, di, s)
                  : bwd_launch<128, false>(mq, mk, mv, mdo, ob, db, lse, prm, di, s);
}

}  // namespace

extern "C" {

int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B,
             int64_t H, int64_t N, int64_t d, int causal, float scale, void* stream) {
    return fwd_impl(q, k, v, o, lse, B, H, N, d, causal, scale, stream, WAIT_LIMIT_NS, 0);
}

int attn_fwd_test_wait_timeout(const void* q, const void* k, const void* v, void* o, float* lse,
                               int64_t B, int64_t H, int64_t N, int64_t d, void* stream) {
    return fwd_impl(q, k, v, o, lse, B, H, N, d, 0, 0.125f, stream, TEST_WAIT_LIMIT_NS, 1);
}

int64_t attn_fwd_schedule(int64_t B, int64_t H, int64_t N, int causal, int grid,
                          int32_t* cta_of_unit, int32_t* slot_of_unit, int64_t capacity) {
    bool empty = false;
    const int st = validate_shape(B, H, N, 128, 1.0f, &empty);
    if (st != ATTN_OK) return st;
    if (empty) return 0;
    if (grid < 1) return ATTN_ERR_SHAPE;
    FwdParams prm;
    memset(&prm, 0, sizeof(prm));
    prm.N = static_cast<int>(N);
    prm.BH = static_cast<int>(B * H);
    prm.n_pairs = static_cast<int>((N + UNIT_ROWS - 1) / UNIT_ROWS);
    prm.nkv = static_cast<int>((N + BLOCK_N - 1) / BLOCK_N);
    prm.n_units = prm.BH * prm.n_pairs;
    if (!cta_of_unit || !slot_of_unit) return ATTN_ERR_NULL;
    if (capacity < prm.n_units) return ATTN_ERR_WORKSPACE;
    if (grid > prm.n_units) grid = prm.n_units;
    plan_schedule(prm, grid);
    for (int64_t i = 0; i < prm.n_units; ++i) cta_of_unit[i] = slot_of_unit[i] = -1;
    int64_t visits = 0;
    for (int c = 0; c < grid; ++c) {
        int slot = 0;
        for (int s = 0;; ++s) {
            Unit u;
            const int got = sched_unit(s, c, grid, causal != 0, prm, u);
            if (got < 0) break;
            if (got == 0) continue;
            ++visits;
            if (u.bh < 0 || u.bh >= prm.BH || u.pair < 0 || u.pair >= prm.n_pairs)
                return ATTN_ERR_SHAPE;   // a unit outside the problem: a scheduling bug
            const int64_t idx = static_cast<int64_t>(u.bh) * prm.n_pairs + u.pair;
            cta_of_unit[idx] = c;
            slot_of_unit[idx] = slot++;
        }
    }
    return visits;
}

size_t attn_fwd_fp8_workspace_bytes(int64_t B, int64_t H, int64_t N, int64_t d) {
    bool empty = false;
    if (validate_shape(B, H, N, d, 1.0f, &empty) != ATTN_OK || empty || B * H > 65535) return 0;
    return fp8_ws_bytes(B * H, N, d);
}

int attn_fwd_fp8(const void* q, const void* k, const void* v, float q_descale, float k_descale,
                 float v_descale, void* o, float* lse, int64_t B, int64_t H, int64_t N, int64_t d,
                 int causal, float scale, void* workspace, size_t workspace_bytes, void* stream) {
    return fp8_impl(q, k, v, q_descale, k_descale, v_descale, o, lse, B, H, N, d, causal, scale,
                    workspace, workspace_bytes, stream);
}

size_t attn_bwd_workspace_bytes(int64_t B, int64_t H, int64_t N, int64_t d) {
    bool empty = false;
    if (validate_shape(B, H, N, d, 1.0f, &empty) != ATTN_OK || empty || B * H > 65535) return 0;
    return bwd_ws_bytes(B * H, N, d);
}

int attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
             const float* lse, void* dq, void* dk, void* dv, int64_t B, int64_t H, int64_t N,
             int64_t d, int causal, float scale, void* workspace, size_t workspace_bytes,
             void* stream) {
    return bwd_impl(q, k, v, o, dout, lse, dq, dk, dv, B, H, N, d, causal, scale, workspace,
                    workspace_bytes, stream, WAIT_LIMIT_NS, 0);
}

int attn_bwd_test_wait_timeout(const void* q, const void* k, const void* v, const void* o,
                               const void* dout, const float* lse, void* dq, void* dk, void* dv,
                               int64_t B, int64_t H, int64_t N, int64_t d, int causal,
                               void* workspace, size_t workspace_bytes, void* stream) {
    return bwd_impl(q, k, v, o, dout, lse, dq, dk, dv, B, H, N, d, causal, 0.125f, workspace,
                    workspace_bytes, stream, TEST_WAIT_LIMIT_NS, 1);
}

size_t attn_standard_workspace_bytes(int64_t B, int64_t H, int64_t N, int64_t d) {
    bool empty = false;
    if (std_validate(B, H, N, d, 1.0f, &empty) != ATTN_OK || empty) return 0;
    return std_ws_bytes(B * H, N);
}

int attn_standard(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B,
                  int64_t H, int64_t N, int64_t d, int causal, float scale, void* workspace,
                  size_t workspace_bytes, void* stream) {
    return std_impl(q, k, v, o, lse, B, H, N, d, causal, scale, workspace, workspace_bytes,
                    stream);
}

static size_t align256(size_t x) { return (x + 255u) & ~static_cast<size_t>(255u); }

size_t attn_fwd_host_workspace_bytes(int64_t B, int64_t H, int64_t N, int64_t d) {
    bool empty = false;
    if (validate_shape(B, H, N, d, 1.0f, &empty) != ATTN_OK) return 0;
    const size_t tbytes = static_cast<size_t>(B * H * N * d) * 2;
    const size_t lbytes = static_cast<size_t>(B * H * N) * 4;
    return 4 * align256(tbytes) + align256(lbytes);
}

int attn_fwd_host(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B,
                  int64_t H, int64_t N, int64_t d, int causal, float scale, void* workspace,
                  size_t workspace_bytes, void* stream) {
    bool empty = false;
    int st = validate_shape(B, H, N, d, scale, &empty);
    if (st != ATTN_OK || empty) return st;
    if (!q || !k || !v || !o || !lse) return ATTN_ERR_NULL;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
        workspace_bytes < attn_fwd_host_workspace_bytes(B, H, N, d))
        return ATTN_ERR_WORKSPACE;
    const int64_t BH = B * H;
    const size_t tbytes = static_cast<size_t>(BH * N * d) * 2;
    const size_t lbytes = static_cast<size_t>(BH * N) * 4;
    char* ws = static_cast<char*>(workspace);
    char* dq = ws;
    char* dk = ws + align256(tbytes);
    char* dv = ws + 2 * align256(tbytes);
    char* dout = ws + 3 * align256(tbytes);
    char* dl = ws + 4 * align256(tbytes);
    const char* hq = static_cast<const char*>(q);
    const char* hk = static_cast<const char*>(k);
    const char* hv = static_cast<const char*>(v);
    char* ho = static_cast<char*>(o);
    char* hl = reinterpret_cast<char*>(lse);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    auto fail = [] { cudaGetLastError(); return ATTN_ERR_CUDA; };

    /* Heads are independent, so the copies and the kernel are pipelined over
     * chunks of heads: chunk c's kernel and copy back run while chunk c+1 is
     * copied in (copies in and out use separate engines).  Small problems take
     * one chunk. */
    constexpr size_t MIN_PIPELINED_BYTES = size_t(32) << 20;
    const int64_t nchunks = (tbytes * 3 < MIN_PIPELINED_BYTES) ? 1 : (BH < 8 ? BH : 8);
    if (nchunks <= 1) {
        if (cudaMemcpyAsync(dq, q, tbytes, cudaMemcpyHostToDevice, s) != cudaSuccess ||
            cudaMemcpyAsync(dk, k, tbytes, cudaMemcpyHostToDevice, s) != cudaSuccess ||
            cudaMemcpyAsync(dv, v, tbytes, cudaMemcpyHostToDevice, s) != cudaSuccess)
            return fail();
        if ((st = attn_fwd(dq, dk, dv, dout, reinterpret_cast<float*>(dl), B, H, N, d, causal,
                           scale, stream)) != ATTN_OK)
            return st;
        if (cudaMemcpyAsync(o, dout, tbytes, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
            cudaMemcpyAsync(lse, dl, lbytes, cudaMemcpyDeviceToHost, s) != cudaSuccess)
            return fail();
        return ATTN_OK;
    }
    int dev = 0;
    DeviceInfo* di = nullptr;
    if ((st = device_info(&dev, &di)) != ATTN_OK) return st;
    // one enqueue sequence at a time per device: the helper streams and events are shared
    static std::mutex host_mutex;
    std::lock_guard<std::mutex> lock(host_mutex);
    {
        std::lock_guard<std::mutex> dlock(g_mutex);
        if (!di->host_ready) {
            for (auto& hs : di->host_streams)
                if (cudaStreamCreateWithFlags(&hs, cudaStreamNonBlocking) != cudaSuccess) return fail();
            for (auto& ev : di->host_events)
                if (cudaEventCreateWithFlags(&ev, cudaEventDisableTiming) != cudaSuccess) return fail();
            di->host_ready = true;
        }
    }
    cudaStream_t s_in = di->host_streams[0], s_k = di->host_streams[1], s_out = di->host_streams[2];
    cudaEvent_t ev_start = di->host_events[0], ev_in = di->host_events[1];
    cudaEvent_t ev_k = di->host_events[2], ev_done = di->host_events[3];
    // everything starts after the work already on the caller's stream
    if (cudaEventRecord(ev_start, s) != cudaSuccess || cudaStreamWaitEvent(s_in, ev_start, 0) != cudaSuccess ||
        cudaStreamWaitEvent(s_k, ev_start, 0) != cudaSuccess ||
        cudaStreamWaitEvent(s_out, ev_start, 0) != cudaSuccess)
        return fail();
    const int64_t per = (BH + nchunks - 1) / nchunks;
    for (int64_t h0 = 0; h0 < BH; h0 += per) {
        const int64_t hn = (BH - h0 < per) ? BH - h0 : per;
        const size_t to = static_cast<size_t>(h0 * N * d) * 2, tn = static_cast<size_t>(hn * N * d) * 2;
        const size_t lo = static_cast<size_t>(h0 * N) * 4, ln = static_cast<size_t>(hn * N) * 4;
        if (cudaMemcpyAsync(dq + to, hq + to, tn, cudaMemcpyHostToDevice, s_in) != cudaSuccess ||
            cudaMemcpyAsync(dk + to, hk + to, tn, cudaMemcpyHostToDevice, s_in) != cudaSuccess ||
            cudaMemcpyAsync(dv + to, hv + to, tn, cudaMemcpyHostToDevice, s_in) != cudaSuccess ||
            cudaEventRecord(ev_in, s_in) != cudaSuccess || cudaStreamWaitEvent(s_k, ev_in, 0) != cudaSuccess)
            return fail();
        if ((st = attn_fwd(dq + to, dk + to, dv + to, dout + to, reinterpret_cast<float*>(dl + lo), 1, hn,
                           N, d, causal, scale, s_k)) != ATTN_OK)
            return st;
        if (cudaEventRecord(ev_k, s_k) != cudaSuccess || cudaStreamWaitEvent(s_out, ev_k, 0) != cudaSuccess ||
            cudaMemcpyAsync(ho + to, dout + to, tn, cudaMemcpyDeviceToHost, s_out) != cudaSuccess ||
            cudaMemcpyAsync(hl + lo, dl + lo, ln, cudaMemcpyDeviceToHost, s_out) != cudaSuccess)
            return fail();
    }
    // the caller's stream continues once the last copy back has finished
    if (cudaEventRecord(ev_done, s_out) != cudaSuccess || cudaStreamWaitEvent(s, ev_done, 0) != cudaSuccess)
        return fail();
    return ATTN_OK;
}

int attn_device_status(void* stream, int reset) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) {
        cudaGetLastError();
        return ATTN_ERR_CUDA;
    }
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_attn_status, sizeof(int)) != cudaSuccess) {
        cudaGetLastError();
        return ATTN_ERR_CUDA;
    }
    if (reset) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(g_attn_status, &zero, sizeof(int)) != cudaSuccess) {
            cudaGetLastError();
            return ATTN_ERR_CUDA;
        }
    }
    return v;
}

const char* attn_status_str(int status) {
    switch (status) {
        case ATTN_OK: return "ok";
        case ATTN_ERR_NULL: return "a required pointer is NULL";
        case ATTN_ERR_ALIGN: return "a device pointer is not 16-byte aligned";
        case ATTN_ERR_HEADDIM: return "head dimension must be 64 or 128";
        case ATTN_ERR_SHAPE: return "B, H or N out of range";
        case ATTN_ERR_SCALE: return "scale must be finite and > 0";
        case ATTN_ERR_DEVICE: return "current device is not an sm_100 (compute capability 10.0) GPU";
        case ATTN_ERR_LAUNCH: return "kernel launch failed";
        case ATTN_ERR_TIMEOUT: return "a bounded wait inside the kernel ran out";
        case ATTN_ERR_CUDA: return "CUDA runtime or driver error";
        case ATTN_ERR_OVERLAP: return "an output buffer overlaps an input or the other output";
        case ATTN_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
        default: return "unknown status";
    }
}

const char* attn_version(void) { return ATTN_VERSION; }

}  // extern "C"

/* Decode with split K/V: its own kernels and entry points. */
#include "attn_decode.cuh"
