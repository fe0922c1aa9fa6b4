/*
 * attn_fwd.h -- C ABI of the B200 (sm_100a) exact-attention forward library.
 *
 * The operation (FlashAttention teaching pages):
 *   "GPU 学习日报 Day 21", section 3.1, states the problem per head:
 *       S = Q K^T / sqrt(d),  P = softmax(S),  O = P V.
 *   Here the score scale is an argument, and an optional causal mask drops key
 *   j from query row i whenever j > i (the same page, section 6 table, row on
 *   causal-mask waste).  The forward pass also returns, per query row, the
 *   statistic the backward pass recomputes from (airsota "science-depth-m4-047",
 *   section 3, point (c)), read as the natural-log log-sum-exp
 *       LSE_i = ln( sum_{j allowed} exp(scale * q_i . k_j) ).
 *   The result is computed as in sections 4-5 of "GPU 学习日报 Day 21": one fused kernel that
 *   tiles Q, K and V through on-chip memory with the online-softmax recurrence,
 *   so the N x N score and probability matrices never reach device memory.
 *
 * Conventions shared by every entry point:
 *   - Tensors are dense and row-major: q, k, v, o are bf16 [B, H, N, d] with d
 *     contiguous; lse is fp32 [B, H, N].  Q, K and V share one sequence length
 *     N (self-attention; the causal mask is aligned at the top-left corner).
 *   - d must be 64 or 128.  B, H, N >= 0; B*H < 2^31; N < 2^31 - 512.  A call
 *     with B*H*N == 0 is not an error: it returns ATTN_OK and launches nothing
 *     (the pointers may then be NULL).
 *   - scale must be finite and > 0 (1/sqrt(d) is the usual choice).
 *   - Device pointers must be 16-byte aligned (the tensor-memory-accelerator
 *     copies require it).  o and lse must not overlap q, k, v or each other.
 *   - The caller owns every buffer.  These calls allocate no device memory.
 *   - stream is a cudaStream_t passed as void*; NULL means the legacy default
 *     stream.  A device call is asynchronous on that stream; a non-zero return
 *     means nothing was launched (or, for attn_fwd_host, that the sequence of
 *     enqueued operations stopped at the failing step).
 *   - Error behaviour: argument errors are detected on the host before any
 *     CUDA call and returned as negative attn_status_t codes.  A device-side
 *     fault (a bounded wait that ran out) is recorded in a per-device status
 *     word that attn_device_status() reads and clears.
 */
#ifndef ATTN_FWD_H
#define ATTN_FWD_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    ATTN_OK = 0,
    ATTN_ERR_NULL = -1,      /* a required pointer is NULL                         */
    ATTN_ERR_ALIGN = -2,     /* a device pointer is not 16-byte aligned            */
    ATTN_ERR_HEADDIM = -3,   /* d is not 64 or 128                                 */
    ATTN_ERR_SHAPE = -4,     /* B, H or N out of range                             */
    ATTN_ERR_SCALE = -5,     /* scale not finite or not > 0                        */
    ATTN_ERR_DEVICE = -6,    /* the current device is not compute capability 10.0  */
    ATTN_ERR_LAUNCH = -7,    /* the kernel launch (or a copy) was refused by CUDA  */
    ATTN_ERR_TIMEOUT = -8,   /* a bounded wait inside the kernel ran out           */
    ATTN_ERR_CUDA = -9,      /* another CUDA runtime/driver error                  */
    ATTN_ERR_OVERLAP = -10,  /* an output buffer overlaps an input or the other one */
    ATTN_ERR_WORKSPACE = -11 /* workspace missing or too small                     */
} attn_status_t;

/*
 * attn_fwd -- fused exact attention forward on device buffers.
 *   q, k, v : device, bf16 [B, H, N, d], read only.
 *   o       : device, bf16 [B, H, N, d], written: O = softmax(scale*QK^T [+mask]) V,
 *             each element rounded once from fp32 to bf16 (round to nearest even).
 *   lse     : device, fp32 [B, H, N], written: LSE_i as defined above.
 *   causal  : 0 = every key attends; non-zero = key j is masked for row i when j > i.
 *   scale   : multiplies q_i . k_j before the softmax.
 * Returns ATTN_OK once the kernel is enqueued on `stream`, else an error code.
 */
int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
             int64_t B, int64_t H, int64_t N, int64_t d, int causal, float scale,
             void* stream);

/*
 * attn_fwd_host_workspace_bytes -- device workspace attn_fwd_host needs for a
 * shape: room for q, k, v, o (bf16) and lse (fp32), each 256-byte aligned.
 * Returns 0 for invalid shapes.
 */
size_t attn_fwd_host_workspace_bytes(int64_t B, int64_t H, int64_t N, int64_t d);

/*
 * attn_fwd_host -- the same operation on HOST buffers: q, k, v are copied into
 * `workspace` (device memory of at least attn_fwd_host_workspace_bytes), the
 * kernel runs there, and O and LSE are copied back into o and lse.  Heads are
 * independent, so above 32 MB of inputs the work is pipelined over up to 8
 * chunks of heads: the copies in, the kernels and the copies back of
 * successive chunks overlap on three helper streams that the library creates
 * on the first such call per device and CUDA context (with four events; the
 * calls of one process enqueue their work one at a time).  All of it starts after the work
 * already on `stream`, and `stream` waits for all of it, so synchronising
 * `stream` covers the call; smaller problems use `stream` alone.  Host buffers
 * should be page-locked for the copies to be asynchronous.  The caller
 * synchronises the stream before reading o and lse.  Same shapes, layouts and
 * error codes as attn_fwd; the host pointers need no alignment.
 */
int attn_fwd_host(const void* q, const void* k, const void* v, void* o, float* lse,
                  int64_t B, int64_t H, int64_t N, int64_t d, int causal, float scale,
                  void* workspace, size_t workspace_bytes, void* stream);

/*
 * attn_device_status -- read the current device's kernel status word after
 * synchronising `stream`: ATTN_OK, or the first device-side error recorded
 * since the last reset (ATTN_ERR_TIMEOUT).  When reset != 0 the word is
 * cleared afterwards.  Returns ATTN_ERR_CUDA if the word cannot be read.
 */
int attn_device_status(void* stream, int reset);

/*
 * attn_bwd_workspace_bytes -- device workspace attn_bwd needs: an fp32 dQ
 * accumulator of B*H*Np*d values (Np = N rounded up to 128) plus two fp32
 * [B, H, Np] vectors, 256-byte aligned pieces.  0 for invalid or empty shapes.
 */
size_t attn_bwd_workspace_bytes(int64_t B, int64_t H, int64_t N, int64_t d);

/*
 * attn_bwd -- gradients of the forward pass with respect to q, k and v, by
 * recomputation from the saved LSE ("science-depth-m4-047", section 3, point
 * (c)): no N x N matrix reaches device memory.  With s_ij = scale q_i . k_j and
 * P_ij = exp(s_ij - LSE_i) (masked j > i when causal):
 *     dV = P^T dO,  dS = P * (dO V^T - D),  D_i = sum_c dO_ic O_ic,
 *     dQ = scale dS K,  dK = scale dS^T Q.
 *   q, k, v, o, dout : device, bf16 [B, H, N, d] (o and lse from attn_fwd with
 *                      the same q, k, v, causal, scale), read only.
 *   lse              : device, fp32 [B, H, N], read only.
 *   dq, dk, dv       : device, bf16 [B, H, N, d], written.
 *   workspace        : device, >= attn_bwd_workspace_bytes, 256-byte aligned,
 *                      caller-owned, contents ignored on entry; calls that
 *                      overlap on the GPU must not share it.
 * A memset and three kernels are enqueued on `stream`.  Same d, scale, alignment and error
 * conventions as attn_fwd; additionally B*H <= 65535, and ATTN_ERR_OVERLAP when dq, dk, dv
 * or the workspace overlap an input or one another.
 */
int attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
             const float* lse, void* dq, void* dk, void* dv, int64_t B, int64_t H, int64_t N,
             int64_t d, int causal, float scale, void* workspace, size_t workspace_bytes,
             void* stream);

/*
 * attn_standard_workspace_bytes -- device workspace attn_standard needs: the
 * N x N score matrix of every head in fp32, rows padded to a multiple of 128
 * (4 * B * H * Np^2 bytes, Np = N rounded up to 128).  0 for invalid shapes.
 */
size_t attn_standard_workspace_bytes(int64_t B, int64_t H, int64_t N, int64_t d);

/*
 * attn_standard -- the same attention computed the standard, unfused way, for
 * comparison with attn_fwd ("GPU 学习日报 Day 21", sections 3.1 and 4.2: three
 * kernels, the N x N matrices written to and read back from device memory).
 * Enqueues on `stream`: S = scale * Q K^T into the workspace (fp32), a row
 * softmax that writes P (bf16, in place) and LSE, and O = P V.  Same layouts,
 * outputs and error codes as attn_fwd, plus: N <= 32768, B*H <= 65535, and a
 * device workspace of at least attn_standard_workspace_bytes (256-byte
 * aligned, caller-owned, contents ignored on entry, not overlapping the
 * inputs or outputs: ATTN_ERR_OVERLAP).
 */
int attn_standard(const void* q, const void* k, const void* v, void* o, float* lse,
                  int64_t B, int64_t H, int64_t N, int64_t d, int causal, float scale,
                  void* workspace, size_t workspace_bytes, void* stream);

/*
 * attn_fwd_fp8_workspace_bytes -- device workspace attn_fwd_fp8 needs: V
 * transposed, B*H*d*Np bytes (Np = N rounded up to 128).  0 for invalid or
 * empty shapes (d must be 64 or 128).
 */
size_t attn_fwd_fp8_workspace_bytes(int64_t B, int64_t H, int64_t N, int64_t d);

/*
 * attn_fwd_fp8 -- the fused forward pass on 8-bit inputs, the FP8 line of the
 * Hopper-era design ("GPU 学习日报 Day 21", section 6): both GEMMs run on the
 * tensor cores with e4m3 operands (tcgen05 kind::f8f6f4) and fp32 accumulators;
 * the softmax and its statistics stay fp32, and P is rounded to e4m3 for P V.
 *   q, k, v : device, e4m3 (OCP FP8 E4M3, 1 byte) [B, H, N, d], read only.  The
 *             attention is that of q*q_descale, k*k_descale, v*v_descale.
 *   q_descale, k_descale, v_descale : finite, > 0 (else ATTN_ERR_SCALE).
 *   o       : device, bf16 [B, H, N, d], written.
 *   lse     : device, fp32 [B, H, N], written (natural log, as attn_fwd).
 *   workspace : device, >= attn_fwd_fp8_workspace_bytes, 256-byte aligned,
 *             caller-owned, contents ignored on entry; it must not overlap the
 *             inputs or outputs (ATTN_ERR_OVERLAP), and calls that overlap on
 *             the GPU must not share it.
 * d is 64 or 128 (ATTN_ERR_HEADDIM otherwise); B*H <= 65535.  Two kernels are
 * enqueued on `stream` (V transposed into the workspace, then the forward
 * kernel).  Otherwise the conventions of attn_fwd.  Rounding P to e4m3 (3
 * mantissa bits) makes |dO| up to 2^-4 * max_j |v_j| per element of O.
 */
int attn_fwd_fp8(const void* q, const void* k, const void* v, float q_descale, float k_descale,
                 float v_descale, void* o, float* lse, int64_t B, int64_t H, int64_t N, int64_t d,
                 int causal, float scale, void* workspace, size_t workspace_bytes, void* stream);

/*
 * attn_decode_workspace_bytes -- device workspace attn_decode needs for a shape
 * ((B*H + 159) partial results of d fp32 values and an (m, l) pair: one per head
 * and CTA that share keys).  Returns 0 for invalid or empty shapes.
 */
size_t attn_decode_workspace_bytes(int64_t B, int64_t H, int64_t N, int64_t d);

/*
 * attn_decode -- attention of ONE new query row per head against N cached keys
 * and values (decoding; "GPU 学习日报 Day 21", section 9 and FAQ Q5), with the
 * key range split across thread blocks and the partial results merged by the
 * online-softmax rule ("Q31：FlashAttention 为什么快", follow-up 3).
 *   q   : device, bf16 [B, H, d] (a [B, H, 1, d] tensor), read only.
 *   k, v: device, bf16 [B, H, N, d], read only.
 *   o   : device, bf16 [B, H, d], written: softmax(scale * q K^T) V (no mask:
 *         the query sees every key).
 *   lse : device, fp32 [B, H], written: ln sum_j exp(scale * q . k_j).
 *   workspace: device scratch of at least attn_decode_workspace_bytes bytes,
 *         256-byte aligned, owned by the caller; its contents on entry are
 *         ignored.  Calls that overlap on the GPU must not share it.
 * Two kernels are enqueued on `stream`: a persistent stream kernel (one CTA per
 * SM, each reading an equal share of the K/V cache once) that writes one partial
 * per (head, CTA) to the workspace, then the combine.  A bounded wait that runs
 * out sets ATTN_ERR_TIMEOUT in the device status word.  Same d, scale,
 * alignment and error conventions as attn_fwd; ATTN_ERR_WORKSPACE when the
 * workspace is missing, misaligned or too small; ATTN_ERR_OVERLAP when o, lse
 * or the workspace overlap an input or one another.
 */
int attn_decode(const void* q, const void* k, const void* v, void* o, float* lse,
                int64_t B, int64_t H, int64_t N, int64_t d, float scale,
                void* workspace, size_t workspace_bytes, void* stream);

/*
 * attn_decode_noalloc -- attn_decode for callers that cannot allocate device
 * memory.  The pages have no counterpart: this entry point exists for callers
 * that may not call cudaMalloc themselves, such as a plugin whose host
 * application owns every device allocation through its own pool, or a
 * latency-bound loop that must not allocate (cudaMalloc can synchronise the
 * device) once it runs.  It takes the same arguments as attn_decode minus the
 * workspace and allocates nothing: the partial results go to a fixed
 * static device buffer inside the library, attn_decode_noalloc_scratch_bytes()
 * = 8 MiB, which every GPU that loads the library holds until the process
 * exits.
 *   - Shapes whose partials need more than that (attn_decode_workspace_bytes
 *     > 8 MiB; about (B*H + 159)*(d + 2)*4 bytes, i.e. any B*H beyond 15972
 *     at d = 128 or 31616 at d = 64) are rejected with ATTN_ERR_WORKSPACE
 *     before anything runs.
 *   - The buffer's device address is looked up on the first call on each
 *     device, with that device current, and again on the first call after
 *     the current CUDA context changed (a cudaDeviceReset, or another context
 *     made current): the address belongs to a context, so a cached one is
 *     never reused in another.  Make such a first call outside any stream
 *     capture.
 *   - Every call shares the one buffer, which keeps the last call's partials.
 *     Nothing in it has to start at zero (every partial is written before it
 *     is read), but calls that overlap on the GPU (other streams, other host
 *     threads) race on it: serialise them.
 */
int attn_decode_noalloc(const void* q, const void* k, const void* v, void* o, float* lse,
                        int64_t B, int64_t H, int64_t N, int64_t d, float scale, void* stream);

/* attn_decode_noalloc_scratch_bytes -- size of the static buffer above (8 MiB). */
size_t attn_decode_noalloc_scratch_bytes(void);

/*
 * attn_fwd_test_wait_timeout -- test hook for failure detection, not an
 * attention call.  Launches the forward kernel (non-causal, same arguments and
 * checks as attn_fwd) with the producer told never to load K and V, and with
 * every bounded wait limited to 20 ms.  The waits run out, the kernel records
 * ATTN_ERR_TIMEOUT in the device status word, frees its tensor memory and
 * exits; o and lse are left unspecified.  No fault or hang is involved and
 * the context stays usable.  Read the outcome with attn_device_status.
 */
int attn_fwd_test_wait_timeout(const void* q, const void* k, const void* v, void* o, float* lse,
                               int64_t B, int64_t H, int64_t N, int64_t d, void* stream);

/*
 * attn_decode_test_wait_timeout -- the same test hook for the decode kernels.
 * Takes attn_decode's arguments minus scale (and the same checks); the loader
 * warp is told never to load K and V and every bounded wait is limited to
 * 20 ms.  The waits run out, ATTN_ERR_TIMEOUT goes to the device status word
 * and the kernels exit; o, lse and the workspace are left unspecified.
 */
int attn_decode_test_wait_timeout(const void* q, const void* k, const void* v, void* o, float* lse,
                                  int64_t B, int64_t H, int64_t N, int64_t d, void* workspace,
                                  size_t workspace_bytes, void* stream);

/*
 * attn_bwd_test_wait_timeout -- the same test hook for the backward pass.
 * Takes attn_bwd's arguments minus scale, with the same checks.  The pre
 * kernel runs as usual.  In the main kernel the TMA warp is told to load
 * nothing (no K, V, Q or dO), and every bounded wait is limited to 20 ms.  The
 * waits run out and ATTN_ERR_TIMEOUT goes to the device status word.  Every
 * CTA then frees its tensor memory and exits.  dq, dk, dv and the workspace
 * are left unspecified.
 */
int attn_bwd_test_wait_timeout(const void* q, const void* k, const void* v, const void* o,
                               const void* dout, const float* lse, void* dq, void* dk, void* dv,
                               int64_t B, int64_t H, int64_t N, int64_t d, int causal,
                               void* workspace, size_t workspace_bytes, void* stream);

/*
 * attn_fwd_schedule -- host-only query of the forward kernel's static work
 * schedule (no CUDA call; usable without a GPU).  The work is split into units
 * of two 128-row Q tiles of one head: unit u = bh * ceil(N/256) + pair covers
 * query rows [256*pair, 256*pair + 256) of head bh.  Persistent CTAs walk the
 * units in a fixed order so that work is spread evenly ("GPU 学习日报 Day 21",
 * section 6: parallelism over query row blocks; longest causal blocks first).
 *   grid          : number of CTAs (attn_fwd uses min(SM count, units)).
 *   cta_of_unit   : host, int32 [capacity], written: the CTA that runs unit u.
 *   slot_of_unit  : host, int32 [capacity], written: u's position in that CTA's
 *                   sequence (0 = first).
 * Returns the number of units the CTAs visit (equal to B*H*ceil(N/256) when
 * every unit runs once), or a negative attn_status_t: ATTN_ERR_SHAPE (shape,
 * grid < 1, or a unit outside the problem), ATTN_ERR_NULL, ATTN_ERR_WORKSPACE
 * (capacity below the unit count).  Head dimension does not change the order.
 */
int64_t attn_fwd_schedule(int64_t B, int64_t H, int64_t N, int causal, int grid,
                          int32_t* cta_of_unit, int32_t* slot_of_unit, int64_t capacity);

/* attn_status_str -- a static, human-readable string for a status code. */
const char* attn_status_str(int status);

/* attn_version -- library version string. */
const char* attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_FWD_H */
