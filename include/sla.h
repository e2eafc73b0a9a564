/*
 * sla.h -- C interface of the SageSLA attention library for NVIDIA B200
 * (sm_100a): INT8 block-quantised, top-k block-sparse softmax attention plus
 * a linear-attention branch for the key blocks that were not selected.
 *
 * The operation is the SageSLA attention module of the pages
 *   [P1] "Turbo Diffusion：秒级生成与高清保真的视频扩散技术突破" (lanhy.cn),
 *        section 三(一) SageAttention2++ items 1-3 and section 三(二) SLA
 *        items 1-3;
 *   [P3] "TurboDiffusion技术指南：突破视频生成效率瓶颈的实践方案"
 *        (blog.gitcode.com), section "SageSLA" and the T2V parameter list
 *        (--attention_type sagesla, --sla_topk 0.1 = keep 10%);
 *   [P4] "TurboDiffusion: 即時AI影片生成的重大突破" (bonega.ai), section
 *        "SLA: 稀疏線性注意力";
 *   [P5] "TuroDiffusion：为高质量视频'系统性提速'" (chooseai.net), the
 *        linear-layer acceleration paragraph (W8A8 on 128x128 blocks).
 * The pages give no formulas; the exact semantics implemented here are:
 *   1. mu = per-channel mean of K over the N tokens (exact sum, rounded once to
 *      float32, for every finite input); K_s = float32(K) - mu.  ([P1] 三(一) item 1, "outlier smoothing")
 *   2. Q and K_s are quantised to INT8 per block of `block` tokens x d channels:
 *      s = max|x| / 127 (float32), code = clamp(round_half_even(x / s), +-127).
 *      ([P1] 三(一) item 2)
 *   3. Block mask: qbar_i, kbar_j = means of the raw Q, K rows of each block
 *      (float64); score = qbar_i . kbar_j / sqrt(d); each query block keeps the
 *      kc = ceil(topk_frac * nblk) key blocks with the largest scores (equal
 *      scores: lower block index first), listed in ascending order.
 *      ([P1] 三(二) item 1; [P3] --sla_topk)
 *   4. For the kept blocks: S = int32(Qi8 . Ki8^T) * sq * sk / sqrt(d),
 *      float32 online softmax, P rounded to bf16, O_sparse = (P . V) / l with
 *      float32 accumulation.  ([P1] 三(一) item 3, 三(二) item 3)
 *   5. For the other blocks: phi = elu + 1 linear attention,
 *      O_lin = phi(q) (sum h_j) / (phi(q) . sum z_j) with per-key-block states
 *      h_j = sum phi(k) v^T, z_j = sum phi(k) of the raw K; none when every
 *      block is kept.  ([P1] 三(二) item 2)
 *   6. out = O_sparse + O_lin . W_proj, formed in float32 and stored as bf16
 *      (round to nearest even; float32 on request).  ([P1] 三(二) item 2,
 *      "linear projection")
 *
 * Conventions for every entry point:
 *   - Tensors are row-major.  q, k, v: bf16 [B, H, N, d] (d innermost); out:
 *     bf16 [B, H, N, d] (float32 through sla_attn_ex).
 *     proj (W_proj): bf16 [d, d], used as O_lin . proj (row vectors).
 *   - All tensor pointers are DEVICE pointers except where an entry point says
 *     HOST.  They must be 16-byte aligned.  The caller owns all memory; the
 *     library never frees or retains caller pointers.
 *   - nblk = ceil(N / block); kc = sla_topk_count(N, block, topk_frac).
 *   - Supported: d in {64, 128}; block in {64, 128}; B, H, N >= 1;
 *     0 < topk_frac <= 1; nblk <= 16384; B*H <= 65535; B*H*nblk*block < 2^31.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Device
 *     entry points only enqueue work on `stream` and return; they may draw
 *     temporary device memory from a library-owned stream-ordered pool.
 *   - Arguments are checked before anything is enqueued; an invalid call
 *     returns an error code and touches no memory.  Faults inside the kernels
 *     surface at the caller's next synchronisation or through
 *     sla_get_error().
 *   - Thread safety: calls are re-entrant, and concurrent calls on different
 *     streams compute independently, with two exceptions: sla_mask_noalloc
 *     calls share one scratch buffer (see there), and the device error word
 *     that sla_get_error() reads is one word per device, not per stream, so a
 *     failure recorded by one stream's kernels is reported to (and cleared by)
 *     whichever caller reads it first.
 */
#ifndef SLA_H_
#define SLA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SLA_OK = 0,
  SLA_ERR_INVALID_ARG = 1,  /* null / misaligned pointer, value out of range     */
  SLA_ERR_UNSUPPORTED = 2,  /* well-formed but outside the supported shapes        */
  SLA_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed                   */
  SLA_ERR_OOM = 4,          /* temporary device memory could not be obtained       */
  SLA_ERR_TIMEOUT = 5,      /* a kernel's bounded wait gave up (sla_get_error)     */
  SLA_ERR_SCRATCH_LIMIT = 7, /* sla_mask_noalloc: the problem needs more scratch than
                               its fixed device buffer holds                       */
  SLA_ERR_SMEM_LAYOUT = 8   /* a kernel's dynamic shared memory did not start on a
                               boundary that leaves room for its aligned tiles; the
                               kernel wrote nothing (sla_get_error)                */
} sla_status;

/* Number of key blocks each query block keeps:
 * clamp(ceil(float(topk_frac) * nblk), 1, nblk), computed exactly in double.
 * Returns -SLA_ERR_INVALID_ARG if N < 1, block < 1 or topk_frac not in (0, 1].
 * Host only; touches no device. */
int sla_topk_count(int N, int block, float topk_frac);

/* Steps 1-2 only (SageAttention2++ smoothing + quantisation, [P1] 三(一) 1-2).
 *   q, k     : in,  bf16 [B,H,N,d]
 *   q_i8     : out, int8 [B,H,nblk*block,d]   codes of Q; rows >= N are 0
 *   k_i8     : out, int8 [B,H,nblk*block,d]   codes of K - mu; rows >= N are 0
 *   q_scale  : out, float [B,H,nblk]
 *   k_scale  : out, float [B,H,nblk]
 *   k_mean   : out, float [B,H,d] (mu), or NULL */
int sla_quant(const void* q, const void* k, int8_t* q_i8, int8_t* k_i8, float* q_scale, float* k_scale,
              float* k_mean, int B, int H, int N, int d, int block, void* stream);

/* Step 3 only (SLA block selection, [P1] 三(二) 1).
 *   blk_idx : out, int32 [B,H,nblk,kc], kept key blocks of each query block, ascending
 *   bitmap  : out, uint8 [B,H,nblk,nblk], 1 where kept, or NULL */
int sla_mask(const void* q, const void* k, int32_t* blk_idx, uint8_t* bitmap, int B, int H, int N, int d,
             int block, float topk_frac, void* stream);

/* Size of the fixed device scratch buffer behind sla_mask_noalloc. */
#define SLA_NOALLOC_SCRATCH_BYTES (16u << 20)

/* sla_mask without any device memory allocation.  The pages have no
 * counterpart to this entry point; it exists for callers that cannot call
 * cudaMalloc or any allocator while they run, for example an inference server
 * that plans every byte of device memory at start-up and forbids allocation
 * afterwards (so that memory use stays predictable and cannot fail with
 * out-of-memory mid-request), or a host that owns the device allocator
 * through another framework.
 *   Arguments, outputs and errors are those of sla_mask.  The block sums the
 * mask needs live in one file-scope device buffer of
 * SLA_NOALLOC_SCRATCH_BYTES (16 MiB) in this library, which every GPU that
 * loads the library holds until the process exits.  A problem must fit in
 * it: 26 * B*H*nblk*d + 4 * B*H*d bytes (nblk rounded up to an even count in
 * 8 * B*H*nblk*d of them), each part rounded up to 256 bytes
 * (for example B*H = 12, nblk = 256, d = 128 fits; B*H = 40, nblk = 591
 * does not); larger ones return SLA_ERR_SCRATCH_LIMIT before any work is
 * enqueued.
 *   The first call on a device looks up the buffer's device address and
 * loads every kernel this entry point can launch (once per device, with that
 * device current; with CUDA's lazy module loading that is where the buffer
 * and the kernels' code are placed on the device); make that first call
 * during start-up, before the caller stops allowing allocation and before any
 * stream capture.  No later call allocates, whatever its shape (keep
 * sla_profile_enable off, its default: profiling creates CUDA events).
 *   All calls on a device share the one buffer and it keeps the last call's
 * contents; every scratch element is written before it is read, so nothing
 * needs clearing.  Calls whose work overlaps on the GPU (for example on two
 * streams without ordering between them) race on the buffer: order them. */
int sla_mask_noalloc(const void* q, const void* k, int32_t* blk_idx, uint8_t* bitmap, int B, int H, int N, int d,
                     int block, float topk_frac, void* stream);

/* The whole operator, steps 1-6 ([P1] 三(二) 3, SageSLA).
 *   q, k, v : in,  bf16 [B,H,N,d]
 *   proj    : in,  bf16 [d,d]
 *   out     : out, bf16 [B,H,N,d], fully overwritten (float32 result rounded
 *             to nearest even)
 * The kernels run on `stream` and on a second stream the library keeps per
 * device (created at the first call), ordered by events: work enqueued on
 * `stream` after the call sees the complete result, and the call can be
 * captured in a CUDA graph.  The second stream is shared by all calls on the
 * device, so the part of concurrent calls that runs there is serialised.
 * (Also sla_attn_ex and sla_attn_classes.) */
int sla_attn(const void* q, const void* k, const void* v, const void* proj, void* out, int B, int H, int N,
             int d, int block, float topk_frac, void* stream);

/* Output element types of sla_attn_ex. */
#define SLA_OUT_BF16 0
#define SLA_OUT_F32 1

/* sla_attn with a choice of output type and, for inspection and tests, the
 * two parts of step 6 on their own:
 *   out       : out, [B,H,N,d] of type out_dtype (SLA_OUT_BF16 or SLA_OUT_F32)
 *   o_sparse  : out, float [B,H,N,d] = O_sparse of step 4, or NULL
 *   o_lin     : out, float [B,H,N,d] = O_lin . W_proj of steps 5-6 (zero when
 *               every block is kept), or NULL
 * Each part asked for costs one more pass of the attention kernel. */
int sla_attn_ex(const void* q, const void* k, const void* v, const void* proj, void* out, int out_dtype,
                float* o_sparse, float* o_lin, int B, int H, int N, int d, int block, float topk_frac,
                void* stream);

/* Finer quantisation granularity ([P1] 三(一) item 2: quantisation parameters
 * per sub-block, "thread level", finer than the attention tiles): one scale
 * per group of `gran` tokens x d channels inside each block (gran = 32, 64 or
 * 128, dividing block; gran = block is the default operator).  Scales are
 * laid out [B,H,nblk*block/gran]; a group wholly past N has scale 0.  The
 * block mask and the linear branch do not depend on it.  Q is not smoothed. */
int sla_quant_gran(const void* q, const void* k, int8_t* q_i8, int8_t* k_i8, float* q_scale, float* k_scale,
                   float* k_mean, int B, int H, int N, int d, int block, int gran, void* stream);
int sla_attn_gran(const void* q, const void* k, const void* v, const void* proj, void* out, int out_dtype,
                  float* o_sparse, float* o_lin, int B, int H, int N, int d, int block, float topk_frac, int gran,
                  void* stream);

/* Three block classes and per-head fractions (an extension: the pages name
 * two classes, the top-K "core" blocks of [P1] 三(二) 1 and the rest through
 * the linear branch of [P1] 三(二) 2; [P4] "SLA: 稀疏線性注意力" replaces dense
 * attention by cheaper substitutes where it is not needed).  Head h (the same
 * h for every batch entry) uses topk_frac[h] and skip_frac[h]:
 *   kc_h = clamp(ceil(float(topk_frac[h]) * nblk), 1, nblk) blocks are kept
 *          (exact attention), as in sla_topk_count;
 *   kn_h = min(floor(float(skip_frac[h]) * nblk), nblk - kc_h) blocks, those
 *          ranked last, are left out of both branches;
 *   the other nblk - kc_h - kn_h blocks go through the linear branch.
 * Ranking: larger pooled score first, equal scores lower block index first
 * (the order sla_mask keeps by).  skip_frac may be NULL (all 0): then every
 * head is the two-class operator with its own fraction.  A query block with
 * no block in the linear branch has no linear part.
 *   topk_frac : in, HOST float [H], each in (0, 1]
 *   skip_frac : in, HOST float [H], each in [0, 1), or NULL
 * H <= 512, else SLA_ERR_UNSUPPORTED. */

/* Host only: kc_h and kn_h for every head (kc, kn: HOST int [H], either may
 * be NULL).  Returns the largest kc_h (the pitch of sla_mask_classes'
 * blk_idx), or minus an error code. */
int sla_head_counts(int N, int block, int H, const float* topk_frac, const float* skip_frac, int* kc, int* kn);

/* Step 3 with per-head counts and three classes.
 *   blk_idx : out, int32 [B,H,nblk,kcp] (kcp = sla_head_counts' result): the
 *             kc_h kept key blocks of each query block, ascending, then -1
 *   classes : out, uint8 [B,H,nblk,nblk]: 2 kept, 1 linear branch, 0 left
 *             out; or NULL */
int sla_mask_classes(const void* q, const void* k, int32_t* blk_idx, uint8_t* classes, int B, int H, int N, int d,
                     int block, const float* topk_frac, const float* skip_frac, void* stream);

/* sla_attn_ex with per-head counts and three classes: the linear branch sums
 * the states of the blocks of class 1 only.  Arguments as sla_attn_ex, with
 * topk_frac and skip_frac as above. */
int sla_attn_classes(const void* q, const void* k, const void* v, const void* proj, void* out, int out_dtype,
                     float* o_sparse, float* o_lin, int B, int H, int N, int d, int block, const float* topk_frac,
                     const float* skip_frac, void* stream);

/* sla_attn on HOST buffers (pageable or pinned): copies q, k, v, proj to the
 * device, runs the operator and copies out (bf16) back, and returns when the
 * result is in host memory.  The (batch, head) pairs are processed in up to
 * six chunks spread over three streams of the current device (created at the
 * first call on that device and kept), so that with pinned host buffers one
 * chunk's copies overlap another chunk's operator (each chunk's kernels stay
 * on that chunk's stream); the result is the same as sla_attn's.  Calls on
 * the same device are serialised. */
int sla_attn_host(const void* q, const void* k, const void* v, const void* proj, void* out, int B, int H,
                  int N, int d, int block, float topk_frac);

/* sla_attn_classes on HOST buffers, as sla_attn_host (output bf16). */
int sla_attn_classes_host(const void* q, const void* k, const void* v, const void* proj, void* out, int B, int H,
                          int N, int d, int block, const float* topk_frac, const float* skip_frac);

/* ---------------------------------------------------------------------------
 * W8A8 linear layer ([P1] 三(四) item 1: weights and activations in 8 bits,
 * quantisation parameters per 128x128 block, activations quantised at run
 * time; [P5] the chooseai.net news page, linear-layer acceleration: both on
 * 128x128 blocks).  Y = X . W^T + bias, X bf16 [M, K], W [N, K] (out_features
 * x in_features), bias bf16 [N] or NULL.
 *   Quantisation of a [R, K] bf16 matrix: blocks of 128 rows x 128 columns
 *   (the last ones partial); per block s = float32(max|x| / 127) and codes
 *   clamp(round_half_even(float32(x / s)), -127, 127) (an all-zero block:
 *   s = 0, codes 0).
 *   Product: Y[m, n] = sum over column blocks kb of P_kb[m, n] *
 *   float32(sx[m/128][kb] * sw[n/128][kb]), P_kb the exact int32 sum of the
 *   int8 products of block kb, accumulated in float32 in kb order, plus
 *   bias[n]; stored as bf16 (round to nearest even) or float32.
 * Supported: M, N, K >= 1, K and N multiples of 16.  Row-major, 16-byte
 * aligned device pointers; `stream` as above. */

/*   x      : in,  bf16 [R, K]
 *   codes  : out, int8 [R, K]
 *   scales : out, float [ceil(R/128), ceil(K/128)] */
int sla_w8a8_quant(const void* x, int R, int K, int8_t* codes, float* scales, void* stream);

/*   xq, sx : in, the codes and scales of X (sla_w8a8_quant)
 *   wq, sw : in, the codes and scales of W (sla_w8a8_quant of W [N, K])
 *   y      : out, [M, N] of type out_dtype (SLA_OUT_BF16 or SLA_OUT_F32) */
int sla_w8a8_gemm(const int8_t* xq, const float* sx, const int8_t* wq, const float* sw, const void* bias, void* y,
                  int out_dtype, int M, int N, int K, void* stream);

/* The layer with the activations quantised in the call (dynamic): X's codes
 * and scales go to temporary memory from the library's stream-ordered pool. */
int sla_w8a8_linear(const void* x, const int8_t* wq, const float* sw, const void* bias, void* y, int out_dtype, int M,
                    int N, int K, void* stream);

/* Synchronises `stream`, then reads and clears the device error word of the
 * current device.  The word is shared by every stream of the device: a code
 * recorded by kernels on another stream is reported here as well, and cleared.
 * Returns SLA_ERR_TIMEOUT if a kernel's bounded wait gave up,
 * SLA_ERR_SMEM_LAYOUT if a kernel could not place its shared-memory tiles,
 * SLA_ERR_CUDA if the synchronisation itself failed, else SLA_OK. */
int sla_get_error(void* stream);

/* Kernel kinds, in the order sla_profile_read() reports them. */
typedef enum {
  SLA_K_STATS = 0,   /* K block sums and linear states              */
  SLA_K_MEAN = 1,    /* per-channel mean of K                        */
  SLA_K_QUANT = 2,   /* smoothing + INT8 quantisation (+ Q block sums) */
  SLA_K_MASK = 3,    /* pooled scores + top-k                        */
  SLA_K_ATTN = 4,    /* critical-block attention + linear part       */
  SLA_K_LINGEMM = 5, /* sums of the non-selected states              */
  SLA_K_QUANT2D = 6, /* W8A8: 128x128 block quantisation             */
  SLA_K_W8A8 = 7,    /* W8A8: block-scaled INT8 GEMM                 */
  SLA_K_COUNT = 8
} sla_kernel_kind;

/* Measurement support (no counterpart on the pages).  While enabled, every
 * kernel the library launches is bracketed by two CUDA events recorded on the
 * stream it runs on.  sla_profile_read() waits for those events, writes per
 * kernel kind the summed device milliseconds (ms[k]) and the number of
 * launches (launches[k]) for k < n (n <= SLA_K_COUNT), and clears them.
 * Either array may be NULL.  Returns SLA_OK or SLA_ERR_CUDA. */
int sla_profile_enable(int on);
int sla_profile_read(double* ms, long long* launches, int n);

/* Failure-path self test (no counterpart on the pages): launches one tiny
 * kernel whose bounded wait on a barrier that nothing completes gives up after
 * its limit (about one second) exactly as a stalled pipeline would: it records
 * SLA_ERR_TIMEOUT in the device error word and returns, leaving the context
 * usable.  Returns SLA_OK once the kernel is enqueued; a following
 * sla_get_error(stream) then reports SLA_ERR_TIMEOUT. */
int sla_selftest_wait_timeout(void* stream);

/* Static description of a status code (never NULL). */
const char* sla_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* SLA_H_ */
