/*
 * strata_moe.h -- C ABI of libstrata_moe.so, the B200 (sm_100a) routed-expert
 * FFN layer of a very sparse mixture-of-experts model.
 *
 * The layer (Strata walk-through, blog.5616760.com/0039, section 5 "MoE 的本质",
 * flowchart "Router -> Top-10 -> softmax 加权合并"): a router scores every
 * token against all experts, the k best experts are chosen, each chosen
 * expert's SwiGLU FFN runs on the token, and the expert outputs are summed
 * with the routing softmax weights.  The pages' geometry is hidden 2560, 512
 * experts per layer, expert width 640, top-10 (lcz.me/topic/2153 section 3.2;
 * ai-coding.wiselychen.com Strata review, "30 秒定位" table); every size here
 * is a runtime argument.
 *
 * Call order for one layer (all on one CUDA stream):
 *   moe_rmsnorm -> moe_router_topk -> moe_bucket -> moe_experts
 *   [-> moe_shared_expert] -> moe_combine
 * or the composite moe_layer_forward, which runs exactly that sequence.
 *
 * Conventions shared by every call
 *   - Every tensor pointer is a DEVICE pointer owned by the caller unless the
 *     argument says otherwise.  The library never allocates, frees or
 *     synchronises device memory (the one exception, strata_read_status, says
 *     so).  Scratch memory comes from a caller-provided `workspace` whose size
 *     the matching *_workspace_size() query returns; its contents need not be
 *     initialised and are clobbered.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Calls are asynchronous: they enqueue kernels and return.
 *   - Return value: a strata_status.  Arguments are validated on the host
 *     before anything is enqueued; on STRATA_EINVAL / STRATA_EUNSUPPORTED
 *     nothing has been enqueued and no output was touched.  STRATA_ECUDA
 *     means a launch failed (cudaGetLastError), outputs are undefined.
 *   - `dev_status` (device int32, may be NULL where stated) is a sticky error
 *     word: kernels never trap; on a device-detected problem (a bounded wait
 *     that ran out, an index out of range) they OR a STRATA_DEV_* bit into it
 *     and skip the offending access; an fp16 intermediate that overflowed
 *     (stored as +-inf) is reported the same way.  Zero it once; read it with
 *     strata_read_status.
 *   - bf16 and fp16 values travel as uint16_t bit patterns.
 *   - Shapes: T tokens, H hidden, E experts, I expert width, k experts per
 *     token, P = T*k (token, slot) pairs; pair p = t*k + j.
 */
#ifndef STRATA_MOE_H
#define STRATA_MOE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define STRATA_API __attribute__((visibility("default")))
#else
#define STRATA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ---------------------------------------------------------------- status */
typedef enum strata_status {
  STRATA_OK = 0,
  STRATA_EINVAL = 1,       /* bad shape, NULL pointer, misalignment, k > E, K % 32 != 0 */
  STRATA_ECUDA = 2,        /* a CUDA launch or API call failed */
  STRATA_EUNSUPPORTED = 3, /* valid but outside what the kernels implement */
  STRATA_ETIMEOUT = 4,     /* device-reported: a bounded wait ran out */
  STRATA_EBOUNDS = 5,      /* device-reported: an index was out of range */
  STRATA_EOVERFLOW = 6     /* device-reported: an fp16 intermediate overflowed */
} strata_status;

/* Bits a kernel ORs into *dev_status. */
#define STRATA_DEV_TIMEOUT 0x1
#define STRATA_DEV_BOUNDS 0x2
/* An fp16 intermediate (the SwiGLU output h of either path, or the prefill
 * expert output y) exceeded the fp16 range and was stored as +-inf. */
#define STRATA_DEV_OVERFLOW 0x4

/* ---------------------------------------------------------------- formats
 * Block-quantised expert weights.  Each weight matrix is stored as
 * output-feature rows with the K (input) dimension contiguous; blocks are 32
 * consecutive K elements of one row with one scale d per block (IEEE fp16,
 * or an E8M0 byte for MXFP4).
 *
 *   STRATA_FMT_Q2_32   2-bit code c in 0..3; w = d * (c - 1.5).
 *                      Codes plane uint8 [N][K/4]: element k is byte k/4,
 *                      bits 2*(k%4) .. 2*(k%4)+1 (least significant first).
 *                      2.5 bits per weight.
 *   STRATA_FMT_Q4CB_32 4-bit code c in 0..15; w = d * KV[c] with the 16-entry
 *                      non-linear codebook
 *                      KV = {-127,-104,-83,-65,-49,-35,-22,-10,
 *                               1,  13, 25, 38, 53, 69, 89,113}
 *                      (the IQ4_NL codebook; the Strata walk-through names
 *                      IQ4_NL in section 13).  Codes plane uint8 [N][K/2]:
 *                      element k is byte k/2, low nibble for even k, high
 *                      nibble for odd k.  4.5 bits per weight.
 *   STRATA_FMT_MXFP4_32 the OCP Microscaling (MX) v1.0 MXFP4 format, in
 *                      which the native-MXFP4 model tier ships its experts
 *                      (lcz.me/topic/2153, model tier list, "ds4f-mxfp4").
 *                      4-bit code c is an FP4 E2M1 number (bit 3 sign, bits
 *                      2-1 exponent with bias 1, bit 0 mantissa, exponent 0
 *                      subnormal: codes 0..7 are 0,0.5,1,1.5,2,3,4,6); the
 *                      block scale is one E8M0 byte e, d = 2^(e-127).
 *                      w = e2m1(c) * d.  Codes plane as for Q4CB_32.
 *                      4.25 bits per weight.  The kernels form w in fp16,
 *                      which is exact for e in 104..140; outside it w is
 *                      fp16-rounded (flushed towards 0 below, +-inf above;
 *                      e = 255, NaN in the format, gives non-finite w).
 *   Scales plane: fp16 [N][K/32], little-endian (Q2_32, Q4CB_32), or
 *   uint8 E8M0 [N][K/32] (MXFP4_32).
 *
 * One expert blob, in this order, every plane starting on a 256-byte boundary:
 *   gate codes [I][H..] | gate scales | up codes [I][H..] | up scales |
 *   down codes [H][I..] | down scales
 * strata_expert_bytes() gives its size: 1,536,000 B for Q2_32 at H=2560,
 * I=640 (the pages' own 2.25-bit Q2_0 blob is 1,382,400 B, lcz.me/topic/2153
 * section 3.4; its bit layout is not on the pages), 2,764,800 B for Q4CB_32
 * at H=2560, I=640 and 14,155,776 B at H=4096, I=2048, 2,611,200 B for
 * MXFP4_32 at H=2560, I=640.  The decode path (T <= STRATA_DECODE_MAX_T)
 * takes MXFP4_32 weights only with H a multiple of 512 (its scale rows are
 * then whole 16-byte units); other H return STRATA_EUNSUPPORTED there. */
#define STRATA_FMT_Q2_32 1
#define STRATA_FMT_Q4CB_32 2
#define STRATA_FMT_MXFP4_32 3

/* Element types of expert outputs y (and of moe_gather_rows rows). */
#define STRATA_DTYPE_F32 0
#define STRATA_DTYPE_F16 1
#define STRATA_DTYPE_BF16 2

/* Largest T served by the weight-streaming decode path of moe_experts;
 * larger T takes the tensor-core grouped-GEMM path. */
#define STRATA_DECODE_MAX_T 16

typedef struct strata_qweights {
  int32_t fmt;            /* STRATA_FMT_* */
  int32_t num_experts;    /* E (1 for a shared expert) */
  int32_t hidden;         /* H, multiple of 128 */
  int32_t inter;          /* I, multiple of 128 */
  const void* base;       /* device; expert e starts at base + e*expert_stride; 256-byte aligned */
  uint64_t expert_stride; /* bytes; multiple of 256 and >= strata_expert_bytes(fmt, H, I) */
} strata_qweights;

/* ---------------------------------------------------------------- helpers */
STRATA_API int32_t strata_abi_version(void);
STRATA_API const char* strata_status_string(int32_t status);
/* Blob size of one expert; 0 for an unknown format or H, I not multiples of 32. */
STRATA_API uint64_t strata_expert_bytes(int32_t fmt, int32_t hidden, int32_t inter);
/* Reads *dev_status (device) into host memory: enqueues a copy on `stream` and
 * SYNCHRONISES that stream.  Returns STRATA_OK, STRATA_ETIMEOUT,
 * STRATA_EBOUNDS, STRATA_EOVERFLOW (the first set bit in that order) or
 * STRATA_ECUDA. */
STRATA_API int32_t strata_read_status(const int32_t* dev_status, void* stream);

/* Failure-detection self-test of the bounded device waits (the pages have
 * no counterpart: it checks this library's own error path).  One CTA runs
 * two of the bounded waits every kernel uses and writes their results
 * (1 = the wait succeeded, 0 = it gave up) to dev_out[0], dev_out[1]:
 *   mode 1: an mbarrier's phase is completed first; the pipeline's
 *           (abort-flag guarded) wait and the epilogue's wait both succeed,
 *           dev_out = {1, 1}, dev_status untouched.
 *   mode 0: nothing arrives on the mbarrier; the first wait gives up after
 *           budget_cycles SM cycles (kernels use about 4e9, 2 s), ORs
 *           STRATA_DEV_TIMEOUT into *dev_status and raises the CTA's abort
 *           flag; the second returns at once; dev_out = {0, 0}.
 *   mode 2: the first wait is the cross-CTA counter wait of the fused decode
 *           kernel, on dev_out[0] (zeroed by the kernel, raised by nobody);
 *           it gives up the same way, the second returns at once;
 *           dev_out = {0, 0}.
 * After a timeout strata_read_status reports STRATA_ETIMEOUT and the context
 * stays usable.  Nothing faults, traps or hangs.
 *   dev_status int32 device word; dev_out int32[2] device.
 *   budget_cycles <= 4e9 and mode in 0..2, else STRATA_EINVAL.
 *   Asynchronous on `stream`. */
STRATA_API int32_t strata_selftest_wait(uint64_t budget_cycles, int32_t mode,
                             int32_t* dev_status, int32_t* dev_out, void* stream);

/* ---------------------------------------------------------------- calls */

/* RMSNorm with unit gain, the layer's input normalisation:
 *   hidden[t,h] = bf16_rne( x[t,h] / sqrt(mean_h x[t,h]^2 + eps) ).
 * x fp32 [T,H] row-major; hidden bf16 [T,H] row-major.  T >= 0 (T == 0 is a
 * no-op), H in 32..16384, multiple of 8.  x and hidden 16-byte aligned. */
STRATA_API int32_t moe_rmsnorm(const float* x, int32_t T, int32_t H, float eps,
                    uint16_t* hidden, void* stream);

/* Router: logits[t,e] = sum_h hidden[t,h]*w_router[h,e] (fp32 accumulation)
 * + bias[e]; p = softmax over all E; the k largest logits are chosen (ties to
 * the lower expert index) and listed in descending-logit order; the weights
 * are renormalised over the chosen k: w_j = p_j / sum_chosen p.
 * (Strata walk-through section 5 flowchart: the router scores each token,
 * top-10 are selected, outputs merged with softmax weights; the Strata review,
 * "success idea one" step 1: the GPU runs the router.)
 *   hidden    bf16 [T,H];  w_router bf16 [H,E] row-major;  bias fp32 [E] or NULL
 *   topk_ids  int32 [T,k] out;  topk_w fp32 [T,k] out
 *   logits_opt fp32 [T,E] out, or NULL
 * Limits: 1 <= k <= min(E, 32); E a multiple of 8, 8..1024; H multiple of 64. */
STRATA_API uint64_t moe_router_topk_workspace_size(int32_t T, int32_t H, int32_t E, int32_t k);
STRATA_API int32_t moe_router_topk(const uint16_t* hidden, const uint16_t* w_router,
                        const float* bias, int32_t T, int32_t H, int32_t E,
                        int32_t k, int32_t* topk_ids, float* topk_w,
                        float* logits_opt, void* workspace, uint64_t ws_bytes,
                        int32_t* dev_status, void* stream);

/* Bucketing of the P = T*k (token, slot) pairs by expert: a deterministic
 * counting sort, stable in pair order (the pages do not name this step; it is
 * what lets one prepared expert weight serve all of its tokens, Strata
 * memory-tier article devotd.net, "读取提示与写出回答时").
 *   counts  int32 [E]     pairs routed to each expert
 *   offsets int32 [E+1]   exclusive prefix sum of counts, offsets[E] = P
 *   perm    int32 [P]     perm[sorted position] = pair p
 *   inv     int32 [P]     inv[p] = sorted position
 *   active  int32 [E+1]   active[0] = U, the number of experts with
 *                         counts > 0; active[1..U] their ids, ascending
 * A topk id outside [0,E) sets STRATA_DEV_BOUNDS and that pair is dropped. */
STRATA_API uint64_t moe_bucket_workspace_size(int32_t T, int32_t k, int32_t E);
STRATA_API int32_t moe_bucket(const int32_t* topk_ids, int32_t T, int32_t k, int32_t E,
                   int32_t* counts, int32_t* offsets, int32_t* perm,
                   int32_t* inv, int32_t* active, void* workspace,
                   uint64_t ws_bytes, int32_t* dev_status, void* stream);

/* The routing step in one call: moe_rmsnorm(x) -> moe_router_topk ->
 * moe_bucket, with the same outputs as those three calls (bit for bit).
 * For T <= STRATA_DECODE_MAX_T (E a multiple of 16, up to 1024) it runs as
 * two kernels over the whole GPU: route_logits (one CTA per 16 experts and
 * slice of H: RMSNorm of the rows, then partial logits from its slice of
 * W_r) and route_select (one CTA: the partial logits summed in a fixed
 * order, + bias, top-k per token, the stable bucket), chained by
 * programmatic dependent launch; other sizes run the three calls.
 *   x      fp32 [T,H];  hidden bf16 [T,H] out (the normalised tokens)
 *   the other arguments as in moe_router_topk and moe_bucket. */
STRATA_API uint64_t moe_route_workspace_size(int32_t T, int32_t H, int32_t E, int32_t k);
STRATA_API int32_t moe_route(const float* x, int32_t T, int32_t H, float eps,
                             const uint16_t* w_router, const float* bias, int32_t E, int32_t k,
                             uint16_t* hidden, int32_t* topk_ids, float* topk_w,
                             int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv,
                             int32_t* active, void* workspace, uint64_t ws_bytes,
                             int32_t* dev_status, void* stream);

/* Routed experts: for every sorted position s with pair p = perm[s], token
 * t = p / k, expert e (offsets[e] <= s < offsets[e+1]):
 *   g = W_gate[e] . hidden[t],  u = W_up[e] . hidden[t],
 *   h = silu(g) * u,            y[s] = W_down[e] . h
 * with fp32 accumulation (the SwiGLU expert FFN; the pages' experts are run by
 * the GPU when resident, Strata review "success idea one" step 2).
 *   y: [P,H] in SORTED order.  T <= STRATA_DECODE_MAX_T: fp32 (decode path,
 *      weight-streaming dequant-GEMV; gate/up and down tiles run in one
 *      kernel, after a one-CTA kernel that zeroes the per-expert counters
 *      it keeps in the workspace, or, where that kernel's shared memory
 *      leaves too few stages, in a gate/up and a down kernel).
 *      T > STRATA_DECODE_MAX_T: fp16 (prefill
 *      path, tcgen05 grouped GEMM over dequantised fp16 tiles).
 *   offsets/perm/active: as written by moe_bucket for the same (T, k, E).
 * Limits: H, I multiples of 128; w->num_experts = E as given to moe_bucket;
 * decode: H a multiple of 256 (512 for MXFP4_32), else STRATA_EUNSUPPORTED;
 * prefill: every code row at least 64 bytes (H and I >= 256 for Q2_32,
 * >= 128 for the 4-bit formats), else STRATA_EUNSUPPORTED.
 * Concurrency (decode path): the fused kernel runs one CTA per SM and its
 * down tiles wait for gate/up tiles of other CTAs, so all its CTAs must be
 * resident together.  Do not run decode moe_experts calls concurrently with
 * other kernels on the device (other streams, other host threads, MPS
 * clients with a share of the SMs): a CTA that cannot become resident
 * leaves the waits of the others to run out, and the call ends with
 * STRATA_DEV_TIMEOUT (after about 2 s) and undefined y. */
STRATA_API uint64_t moe_experts_workspace_size(const strata_qweights* w, int32_t T, int32_t k);
STRATA_API int32_t moe_experts(const uint16_t* hidden, const strata_qweights* w,
                    const int32_t* offsets, const int32_t* perm,
                    const int32_t* active, int32_t T, int32_t k, void* y,
                    void* workspace, uint64_t ws_bytes, int32_t* dev_status,
                    void* stream);

/* moe_experts on the decode path (T <= STRATA_DECODE_MAX_T) without a
 * workspace argument.  The paper has no counterpart of this call.  It is for
 * callers that cannot give the library device memory: a plain-C host with no
 * device allocator of its own, or a process that has already claimed all free
 * HBM (weights plus a cache pool), where a cudaMalloc during a step would fail
 * and a cudaFree would synchronise the device.  The call allocates nothing (no
 * cudaMalloc, cudaFree or allocating library routine); its scratch, the fp16
 * activations h [T*k, I] (up to 2 MiB) and T*k progress counters, lives in one
 * file-scope array of the library.
 *   Limit: T <= STRATA_DECODE_MAX_T and T*k*I <= 1,048,576 (2 MiB of fp16);
 *   beyond it the call returns STRATA_EUNSUPPORTED and launches nothing.
 *   Set-up: the first call on each device, with that device current, looks
 *   up the array's device address (cudaGetSymbolAddress) and caches it for
 *   that device and its current CUDA context (a new context, e.g. after
 *   cudaDeviceReset, looks it up again); make that first call before any
 *   stream capture.  A failed lookup returns STRATA_ECUDA.
 *   Sharing: all calls on a device use the same array, which keeps the last
 *   call's contents; no part of it has to start at zero (each call zeroes its
 *   counters before use and reads only the h rows it wrote).  Calls that
 *   overlap on the GPU (other streams, other host threads) race on the
 *   array: serialise them.
 * Other arguments, the output y (fp32 [T*k, H], sorted order) and the other
 * errors are those of moe_experts. */
STRATA_API int32_t moe_experts_static_scratch(const uint16_t* hidden, const strata_qweights* w,
                                   const int32_t* offsets, const int32_t* perm,
                                   const int32_t* active, int32_t T, int32_t k, float* y,
                                   int32_t* dev_status, void* stream);

/* Shared expert: the same SwiGLU FFN with one always-on expert (w->num_experts
 * == 1) applied to every token, y[t] = FFN(hidden[t]); y [T,H] in token order,
 * fp32 for T <= STRATA_DECODE_MAX_T, fp16 otherwise.  The shared expert is
 * resident and read for every token (Strata review, Table 1 of the paper it
 * quotes; devotd.net memory-tier article, "各层内存承担的数据"). */
STRATA_API uint64_t moe_shared_expert_workspace_size(const strata_qweights* w, int32_t T);
STRATA_API int32_t moe_shared_expert(const uint16_t* hidden, const strata_qweights* w,
                          int32_t T, void* y, void* workspace, uint64_t ws_bytes,
                          int32_t* dev_status, void* stream);

/* Weighted combine ("softmax 加权合并", Strata walk-through section 5), in a
 * fixed order so the result is deterministic:
 *   acc = sum_{j=0..k-1} topk_w[t,j] * y[inv[t*k+j]]   (fp32, j ascending)
 *   acc += shared_y[t]                                 (if shared_y != NULL)
 *   out[t] = bf16_rne(acc);  residual_out[t] = residual[t] + acc  (if given)
 *   y        [P,H] sorted order, y_dtype STRATA_DTYPE_F32 or _F16
 *   shared_y [T,H] or NULL, shared_dtype as y_dtype
 *   residual fp32 [T,H] or NULL (required if residual_out != NULL)
 *   out      bf16 [T,H];  residual_out fp32 [T,H] or NULL (may alias residual)
 * H multiple of 8; all row pointers 16-byte aligned.
 * The kernel is a programmatic dependent launch: it reads inv, topk_w and
 * residual before waiting for the preceding kernel of the stream, and y and
 * shared_y after.  So inv, topk_w and residual must not be written by the
 * immediately preceding kernel if that kernel releases its dependents early
 * (griddepcontrol.launch_dependents); this library's expert kernels write
 * only y / shared_y, and ordinary kernels release nothing early. */
STRATA_API int32_t moe_combine(const void* y, int32_t y_dtype, const int32_t* inv,
                    const float* topk_w, const void* shared_y,
                    int32_t shared_dtype, const float* residual, int32_t T,
                    int32_t k, int32_t H, uint16_t* out, float* residual_out,
                    int32_t* dev_status, void* stream);

/* Row gather, the data movement of expert parallelism (the pages mention
 * experts on several GPUs, lcz.me/topic/2153 "path D" list; they give no
 * kernel for it):  dst[i] = src[idx[i] / div] for i < n.
 *   src   [n_src, H] rows of src_dtype; dst [n, H] rows of dst_dtype
 *   idx   int32 [n]; an index outside [0, n_src*div) sets STRATA_DEV_BOUNDS
 *         and that row of dst is written as zeros
 *   div   >= 1 (k: the hidden rows of (token, slot) pairs in sorted order,
 *         idx = perm; 1: rows put back in another order, idx = inv)
 *   dtypes STRATA_DTYPE_F32 / _F16 / _BF16; dst_dtype == src_dtype, or
 *         src F16 -> dst F32 (exact widening)
 * H a multiple of 8; src and dst 16-byte aligned.  n == 0 is a no-op. */
STRATA_API int32_t moe_gather_rows(const void* src, int32_t src_dtype, int32_t n_src,
                                   int32_t H, const int32_t* idx, int32_t div, int32_t n,
                                   void* dst, int32_t dst_dtype, int32_t* dev_status,
                                   void* stream);

/* The whole layer in one call: moe_rmsnorm(x) -> moe_router_topk ->
 * moe_bucket -> moe_experts -> moe_shared_expert (if `shared` != NULL) ->
 * moe_combine(residual = x).  Every intermediate lives in `workspace`.
 *   x            fp32 [T,H]  layer input (the residual stream)
 *   w_router     bf16 [H,E]; bias fp32 [E] or NULL
 *   w            routed experts (num_experts = E); shared: NULL or one expert
 *   out          bf16 [T,H]  the MoE output, before the residual add
 *   residual_out fp32 [T,H] or NULL: x + MoE output (may alias x)
 *   topk_ids_opt int32 [T,k] / topk_w_opt fp32 [T,k]: copies of the routing,
 *                or NULL */
STRATA_API uint64_t moe_layer_workspace_size(int32_t T, int32_t E, int32_t k,
                                  const strata_qweights* w,
                                  const strata_qweights* shared);
STRATA_API int32_t moe_layer_forward(const float* x, int32_t T, const uint16_t* w_router,
                          const float* bias, int32_t E, int32_t k,
                          const strata_qweights* w, const strata_qweights* shared,
                          float eps, uint16_t* out, float* residual_out,
                          int32_t* topk_ids_opt, float* topk_w_opt,
                          void* workspace, uint64_t ws_bytes,
                          int32_t* dev_status, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* STRATA_MOE_H */
