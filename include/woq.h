/*
 * woq.h -- C ABI of libwoq: weight-only block-32 int4/int8 quantised matmul on B200 (sm_100a).
 *
 * What is computed. Weights W [n, k] (out, in) are stored packed as symmetric signed
 * integers in blocks of 32 consecutive values along k, one IEEE binary16 scale per block;
 * activations and results are FP32 and the products accumulate in FP32; dequantisation is
 * fused into the multiply and no dequantised weight tensor is ever written. The pages
 * this follows:
 *   - "TinyMOSS-Diarize" (devpost), "How we built it": strictly weight-only kernels, FP32
 *     activations, dequantisation fused into the matmul, no materialised dequantised
 *     weights; a blocked GEMM path for prefill and a separate GEMV path for decode; packed
 *     tensors in a container whose tensor table is 64-byte aligned.
 *   - "MOSS-Transcribe-Diarize -- LiteRT (TFLite)", "Files": the production decoder is
 *     int4 in blocks of 32 ("q4b32").
 *   - "MOSS Transcribe Diarize 0.9B" (soniqo, Russian guide), "Implementation notes":
 *     symmetric linear INT8 quantisation with block 32 for the decoder.
 *   - "MOSS Transcribe Diarize 0.9B" (soniqo, English guide), "INT5 vs INT8": names a 5-bit
 *     width beside INT8 but no format; the int5 layout below is this library's own.
 *
 * Packed layout (fixed; qpack produces it bit-exactly):
 *   bits == 4: row r of W occupies k/2 bytes at packed + r*k/2. Byte j holds element 2j in
 *              bits 0-3 and element 2j+1 in bits 4-7, each a 4-bit two's-complement code
 *              in [-8, 7].
 *   bits == 8: row r occupies k bytes at packed + r*k, one two's-complement byte per
 *              element, codes in [-128, 127].
 *   bits == 5: (k % 128 == 0) row r occupies 5k/8 bytes at packed + r*5k/8, codes in
 *              [-16, 15], scale max|w|/15. The first k/2 bytes hold each code's low four
 *              bits laid out as bits == 4 does; then k/32 little-endian 32-bit words, word b
 *              holding bit 4 of block b's codes: element e (0..31) of the block at bit
 *              e/8 + 4*(e%4) + 16*((e%8)/4), so that one shift and mask per 8 codes lines
 *              the fifth bits up with the low nibbles of a 32-bit load.
 *   scales:    binary16 bit patterns, [n, k/32] row-major; element (r, j) scales codes
 *              k in [32j, 32j+32) of row r. W_hat[r, c] = scale[r, c/32] * code[r, c].
 *   All codes a container may hold are decoded, including -8 / -16 / -128, which qpack never
 *   emits.
 *
 * Conventions for every call:
 *   - Return WOQ_OK (0) or a negative WOQ_E* status; arguments are checked before any
 *     work is queued, and a failed check queues nothing.
 *   - Device pointers are CUDA device addresses on the current device; the caller owns
 *     every buffer and the stream. The library allocates no memory and never
 *     synchronises the stream; results are ready when the caller's stream reaches them.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).
 *   - Kernel faults, if any, surface at the caller's next synchronisation.
 */
#ifndef WOQ_H
#define WOQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes. */
#define WOQ_OK          0
#define WOQ_EINVAL     -1  /* null pointer, bits not 4/5/8, block not 32, m out of range,    */
                           /* bad path, or a path that does not take int5                 */
#define WOQ_ESHAPE     -2  /* n or k <= 0, k % 32 != 0, or a size above a documented limit    */
#define WOQ_EALIGN     -3  /* packed/scales not 64-byte aligned, or x/y not 16-byte aligned    */
#define WOQ_ERANGE     -4  /* qpack: non-finite weight, or a block scale overflows binary16    */
#define WOQ_EDEVICE    -5  /* the current device is not compute capability 10.0 (B200)        */
#define WOQ_ECUDA      -6  /* a CUDA runtime call or kernel launch failed                     */
#define WOQ_ETIMEOUT   -7  /* a bounded device-side wait gave up (see woq_device_status)      */
#define WOQ_EWORKSPACE -8  /* qgemm: workspace null or smaller than qgemm_workspace_bytes     */

/* qgemm paths. */
#define WOQ_PATH_AUTO     0  /* by m: BF16_TC, SPLIT_TC or FP32 (see qgemm)                */
#define WOQ_PATH_FP32     1  /* FP32 products and accumulation (CUDA cores), exact codes      */
#define WOQ_PATH_BF16_TC  2  /* tcgen05 tensor cores on bf16(X) and bf16(scale*code)          */
#define WOQ_PATH_SPLIT_TC 3  /* tcgen05 tensor cores, FP32-accurate: X and scale*code each as  */
                             /* bf16 hi + bf16 lo, three products (lo*lo, below 2^-16 of each */
                             /* term, dropped) accumulated in FP32                            */

/*
 * One packed weight [n, k] in device memory.
 *   bits    4, 5 or 8 (5: k % 128 == 0)
 *   block   must be 32
 *   n, k    rows (out features) and columns (in features); k % 32 == 0
 *   packed  device pointer, 64-byte aligned, n*k*bits/8 bytes in the layout above
 *   scales  device pointer, 64-byte aligned, n*(k/32) binary16 bit patterns
 */
typedef struct woq_weight {
  int32_t bits;
  int32_t block;
  int64_t n;
  int64_t k;
  const uint8_t *packed;
  const uint16_t *scales;
} woq_weight;

/*
 * qpack -- host-side quantiser (all pointers are HOST memory; no GPU is used).
 * Follows the formats of "MOSS-Transcribe-Diarize -- LiteRT (TFLite)", "Files" (q4b32) and
 * the soniqo Russian guide, "Implementation notes" (symmetric INT8 block-32). For each row
 * r and block j:
 *   a = max |W[r, 32j .. 32j+31]|                                  (exact, over the floats)
 *   s = binary16 round-half-even of (double)a / qmax, qmax = 7 (int4), 15 (int5) or 127 (int8)
 *   q = clamp(round-half-even((double)w / (double)s), -2^(bits-1), 2^(bits-1)-1), or 0 if s == 0
 * and writes q into `packed` and the bit pattern of s into `scales`, in the layout above.
 *   W       [n, k] float32, row-major
 *   packed  out, n*k*bits/8 bytes;  scales  out, n*(k/32) uint16
 * Errors: WOQ_EINVAL (null pointer, bits), WOQ_ESHAPE (n, k), WOQ_ERANGE (a non-finite W,
 * or a scale that rounds to infinity: a/qmax >= 65520). On error the outputs may be
 * partially written.
 */
int qpack(const float *W, int64_t n, int64_t k, int32_t bits, uint8_t *packed, uint16_t *scales);

/*
 * qgemv -- decode path, y[m, n] = x[m, k] . W_hat^T for 1 <= m <= 64 ("TinyMOSS-Diarize",
 * "How we built it": the separate GEMV path for decode). FP32 accuracy: within a 32-block
 * the codes are multiplied exactly and the block sum is scaled once, in FP32 (CUDA-core and
 * WOQ_GEMV_SPLIT_TC forms), or x and s*q go to the tcgen05 tensor cores as bf16 hi + lo pairs
 * (WOQ_GEMV_SPLIT_GEMM), or the codes and x's signed digits go to the integer tensor cores
 * (WOQ_GEMV_INT8_TC). The kernel is chosen by shape, as measured on B200: on matrices wide
 * enough that 128-row tiles cover every SM (n / 128 >= SM count), m <= 2 the CUDA-core form,
 * 3 <= m <= 4 WOQ_GEMV_INT8_TC for int8 and WOQ_GEMV_SPLIT_TC for int4, up to m = 32
 * WOQ_GEMV_SPLIT_TC, from m = 33 WOQ_GEMV_SPLIT_GEMM; on narrower matrices the CUDA-core form
 * below m = 16 and WOQ_GEMV_SPLIT_GEMM from there; int5 always the CUDA-core form.
 * Deterministic: the same inputs give the same bits on every call. For int5 at m = 1 the
 * CUDA-core form may split each row's k (k > 1024) across 2 or 4 warps and add their sums
 * in a fixed order, so such a row can differ in the last bits from the same row computed in
 * a batch; at one m, qgemv, qgemv_argmax and qgemv_residual add in the same order.
 *   x  device, [m, k] float32 row-major, 16-byte aligned
 *   w  host pointer to the weight descriptor (read during the call only)
 *   y  device, [m, n] float32 row-major, 16-byte aligned; fully overwritten
 * Limits: k <= 32768 (the x rows are staged in shared memory); int5 k <= 10752 (its only
 * kernel stages one x row beside a stage of 8 weight rows in 100 KB; at m = 1 over few rows
 * a 4-row split-K stage can take somewhat more). Errors: WOQ_EINVAL,
 * WOQ_ESHAPE, WOQ_EALIGN, WOQ_EDEVICE, WOQ_ECUDA.
 */
int qgemv(const float *x, int64_t m, const woq_weight *w, float *y, void *stream);

/*
 * qgemv_path -- qgemv with the kernel named instead of chosen by shape.
 *   WOQ_GEMV_AUTO       as qgemv
 *   WOQ_GEMV_CUDA_CORE  FP32 products and FP32 accumulation on the CUDA cores
 *   WOQ_GEMV_SPLIT_TC   tensor cores: each x value is split into bf16 hi + bf16 lo
 *                       (x - hi, rounded), the codes (exact in bf16) are multiplied against
 *                       both in bf16 x bf16 -> FP32 MMAs, and each 32-block's FP32 sum is
 *                       scaled by its binary16 scale in FP32. The split keeps 16 of x's 24
 *                       significand bits; error stays within the FP32 tolerance of qgemv.
 *                       Needs 2 <= m <= 64, k % 256 == 0 and k <= 8192, else WOQ_ESHAPE.
 *   WOQ_GEMV_SPLIT_GEMM the tcgen05 split GEMM of qgemm's WOQ_PATH_SPLIT_TC (x and s*q each
 *                       as bf16 hi + lo, products in an FP32 tensor-memory accumulator,
 *                       64-row tiles); no workspace. Any 1 <= m <= 64.
 *   WOQ_GEMV_INT8_TC    the integer tensor cores (tcgen05 kind::i8), following
 *                       "TinyMOSS-Diarize", "What's next" (an i8mm path that does not quantise
 *                       the activations): per activation row and 32-block, x is written
 *                       exactly enough as 2^E (d0 + d1 2^-7 + d2 2^-14) with integer digits
 *                       |d_i| <= 64 and the block's own power-of-two exponent E (remainder
 *                       below 2^-20 of the block's largest |x|); the codes (int8 as they are,
 *                       int4 times 16) are multiplied by each digit exactly in int32, one sum
 *                       per block, and the block sums are scaled by 2^E and the binary16 scale
 *                       and accumulated in FP32. K-splits of a 128-row tile run as one
 *                       thread-block cluster and are summed in shared memory in a fixed order.
 *                       Needs 1 <= m <= 4 and k % 128 == 0, else WOQ_ESHAPE. A block holding a
 *                       non-finite x makes the outputs it feeds NaN.
 * Arguments and errors otherwise as qgemv; an unknown path is WOQ_EINVAL.
 */
#define WOQ_GEMV_AUTO       0
#define WOQ_GEMV_CUDA_CORE  1
#define WOQ_GEMV_SPLIT_TC   2
#define WOQ_GEMV_SPLIT_GEMM 3
#define WOQ_GEMV_INT8_TC    4
int qgemv_path(const float *x, int64_t m, const woq_weight *w, float *y, int32_t path,
               void *stream);

/*
 * qgemv_swiglu -- a fused gate|up projection and its SwiGLU: with W's rows interleaved
 * (row 2i the gate row i, row 2i+1 the up row i; n = 2I), y[j, i] = silu(g) * u where
 * g = (x . W_hat^T)[j, 2i], u = (x . W_hat^T)[j, 2i+1] and silu(g) = g / (1 + exp(-g)), the
 * Qwen3-style MLP activation the decoder's feed-forward uses. The 2I projection outputs are
 * never written. g and u are computed exactly as qgemv's CUDA-core form computes them.
 *   x  device, [m, k] float32 row-major, 16-byte aligned, 1 <= m <= 64
 *   w  host pointer to the weight descriptor; n even (rows interleaved as above)
 *   y  device, [m, n/2] float32 row-major; fully overwritten
 * Limits: k <= 8192; k <= 4096 always fits, larger k while a stage of 16 weight rows and the
 * x rows of a CTA fit in the kernel's shared-memory budget (int4 up to 7168), else
 * WOQ_ESHAPE. Errors: as qgemv, and WOQ_ESHAPE for an odd n.
 */
int qgemv_swiglu(const float *x, int64_t m, const woq_weight *w, float *y, void *stream);

/*
 * qgemv_residual -- a decode projection with the residual add fused: y[j, i] = (x . W_hat^T)[j, i]
 * + r[j, i], one FP32 add after the projection, which is computed exactly as qgemv's CUDA-core
 * form computes it. In a Qwen3-style decoder block the attention output projection and the
 * MLP down projection each add their result to the residual stream; with r == y the call
 * updates that stream in place (hidden += o_proj(attn)).
 *   x  device, [m, k] float32 row-major, 16-byte aligned, 1 <= m <= 64
 *   w  host pointer to the weight descriptor (read during the call only)
 *   r  device, [m, n] float32 row-major, 4-byte aligned; may be y itself
 *   y  device, [m, n] float32 row-major, 4-byte aligned; fully overwritten
 * Limits: k <= 8192; k <= 4096 always fits, larger k while one stage of weight rows and the
 * x rows of a CTA fit in the kernel's shared-memory budget (int4 up to 8192, int8 up to 7680),
 * else WOQ_ESHAPE. Errors: as qgemv, and WOQ_EINVAL if r and y overlap without being equal.
 */
int qgemv_residual(const float *x, int64_t m, const woq_weight *w, const float *r, float *y,
                   void *stream);

/*
 * qgemv_argmax -- greedy pick over a GEMV's outputs without writing them: for each activation
 * row i, idx[i] = the smallest j with y[i, j] = max over j of y[i, j], and val[i] = that
 * maximum, where y = x . W_hat^T is computed exactly as qgemv's CUDA-core form computes it.
 * Meant for the tied lm_head at decode under greedy decoding (the soniqo guide, Russian
 * edition, "Заметки реализации": its runtime decodes greedily): the 151,936 logits are
 * never written. A NaN output counts as the maximum. Deterministic.
 *   x    device, [m, k] float32 row-major, 16-byte aligned, 1 <= m <= 8
 *   w    host pointer to the weight descriptor (read during the call only)
 *   idx  device, [m] int64, 8-byte aligned; used as scratch during the call, then the index
 *   val  device, [m] float32; the maximum
 * Limits: k <= 8192 and n < 2^31; k <= 4096 always fits, larger k while one stage of weight
 * rows and the x rows of a CTA fit in the kernel's shared-memory budget (int4 up to 8192,
 * int8 up to 7680). Errors: as qgemv, and WOQ_ESHAPE for shapes the fused kernel does not
 * cover.
 */
int qgemv_argmax(const float *x, int64_t m, const woq_weight *w, int64_t *idx, float *val,
                 void *stream);

/*
 * qgemv_chain -- a decode step's GEMVs as one persistent launch, in order ("TinyMOSS-Diarize",
 * "What we learned": match the threading granularity to the size of the operation; a decoder
 * block's projections at one token are each too small to fill the GPU). Item i computes
 *   WOQ_EPI_NONE      y = x . W_hat^T                         y [m, n]
 *   WOQ_EPI_SWIGLU    y[j, i] = silu(g) * u over rows 2i (gate), 2i+1 (up), as qgemv_swiglu
 *                                                             y [m, n/2]
 *   WOQ_EPI_RESIDUAL  y = x . W_hat^T + r, r may be y itself  y [m, n]
 * with the arithmetic of qgemv's CUDA-core form (exact codes, each 32-block's FP32 sum scaled
 * once by its binary16 scale, FP32 accumulation; when a row's K is split across warps, the
 * parts are added in a fixed order). Item i reads its x (and r) only after every earlier
 * item's outputs are complete, so an input may be an earlier item's output: the launch keeps
 * the order that separate calls on one stream would have. Deterministic.
 *   items     host array of `count` descriptors (read during the call only), 1 <= count <= 8
 *   m         activation rows, 1 <= m <= 8
 *   workspace device, 256-byte aligned, >= qgemv_chain_workspace_bytes() bytes: counters that
 *             must be zero before the first call; every call that returns WOQ_OK leaves them
 *             zero again (after a WOQ_ETIMEOUT from woq_device_status, zero them before reuse).
 *             Calls sharing one workspace must be ordered on one stream.
 * Each item: w as for qgemv with k % 256 == 0 and k <= 8192 (the x rows, m rounded up to 1,
 * 2, 4 or 8 of them at the largest k, are staged in each CTA's shared memory beside at least
 * two weight stages: every k fits at m <= 4, at m = 8 up to about 5600; WOQ_ESHAPE beyond);
 * x [m, k] and y device, 16-byte
 * aligned, y not overlapping x; r (WOQ_EPI_RESIDUAL only) device, 16-byte aligned, equal to y
 * or not overlapping it. Errors: WOQ_EINVAL, WOQ_ESHAPE, WOQ_EALIGN, WOQ_EWORKSPACE,
 * WOQ_EDEVICE, WOQ_ECUDA. The launch holds one CTA per SM, and its CTAs wait for one another
 * between items (bounded waits: a wait that gives up is reported by woq_device_status).
 */
#define WOQ_EPI_NONE       0
#define WOQ_EPI_SWIGLU     1
#define WOQ_EPI_RESIDUAL   2
#define WOQ_CHAIN_MAX_ITEMS 8
typedef struct woq_chain_item {
  const woq_weight *w;
  const float *x;
  float *y;
  const float *r;
  int32_t epilogue;
} woq_chain_item;
size_t qgemv_chain_workspace_bytes(void);
int qgemv_chain(const woq_chain_item *items, int32_t count, int64_t m, void *workspace,
                size_t workspace_bytes, void *stream);

/*
 * Bytes of device workspace qgemm needs for (m, w, path); 0 if none. Returns 0 for
 * invalid arguments too (qgemm itself reports those).
 */
size_t qgemm_workspace_bytes(int64_t m, const woq_weight *w, int32_t path);

/*
 * qgemm -- prefill path, Y[m, n] = X[m, k] . W_hat^T for any m >= 1 ("TinyMOSS-Diarize",
 * "How we built it": the blocked GEMM path for prefill, each weight tile unpacked once
 * and reused across activation rows).
 *   path WOQ_PATH_BF16_TC: X is rounded to bf16 into the workspace, each weight tile is
 *        dequantised once into shared memory as bf16(scale*code) and multiplied on the
 *        tcgen05 tensor cores with FP32 accumulation in tensor memory.
 *   path WOQ_PATH_SPLIT_TC: FP32 accuracy on the tcgen05 tensor cores. Each x value is
 *        split into hi = bf16(x) and lo = bf16(x - hi), and each dequantised weight
 *        v = scale*code (exact in FP32) into hi = bf16(v) and lo = bf16(v - hi); the tiles
 *        hold 64 activation rows, and one MMA per operand half multiplies the weight tile
 *        against both X halves, so all four products land in the FP32 accumulator. For
 *        int4, v_hi + v_lo == v exactly; x (and an int8 v) keeps 16 significand bits.
 *        Four times the tensor-core work of BF16_TC; meant for small batches whose FP32
 *        CUDA-core cost grows with m. One launch, no workspace (qgemm_workspace_bytes is 0):
 *        the kernel converts X itself, and when K is split across CTAs those CTAs form one
 *        thread-block cluster that sums the partials in shared memory, in a fixed order.
 *   path WOQ_PATH_FP32: the same FP32 arithmetic as qgemv, for any m.
 *   path WOQ_PATH_AUTO: BF16_TC if m >= 128, SPLIT_TC if 16 <= m < 128, else FP32 (int5:
 *        always FP32).
 *   X  device, [m, k] float32 row-major, 16-byte aligned
 *   Y  device, [m, n] float32 row-major, 16-byte aligned; fully overwritten
 *   workspace  device, 256-byte aligned, at least qgemm_workspace_bytes(m, w, path) bytes
 *              (may be NULL when that is 0); its contents on entry do not matter, and
 *              calls sharing one workspace must be ordered on one stream
 * Errors: WOQ_EINVAL, WOQ_ESHAPE, WOQ_EALIGN, WOQ_EDEVICE, WOQ_EWORKSPACE, WOQ_ECUDA.
 * If a bounded wait gives up inside the tensor-core kernel, the kernel records the event,
 * drains its in-flight copies and MMAs, frees its tensor memory and returns, leaving Y
 * unspecified; woq_device_status reports it.
 */
int qgemm(const float *X, int64_t m, const woq_weight *w, float *Y, int32_t path,
          void *workspace, size_t workspace_bytes, void *stream);

/*
 * qgemm_bf16_noalloc -- the WOQ_PATH_BF16_TC qgemm for callers that cannot allocate device
 * memory. The pages have no counterpart to this call; it exists for integration.
 * Who needs it: a caller that can pass its input and output buffers but has no way to
 * obtain a workspace -- a plugin whose host hands it only its tensors, a serving runtime
 * that has reserved all device memory for its own pool and forbids other allocations, or
 * a latency-critical loop that cannot afford cudaMalloc's implicit device-wide
 * synchronisation.
 * Instead of a caller workspace it uses one fixed 32 MiB scratch array compiled into the
 * library (a __device__ symbol; every GPU that loads the library holds it until the
 * process exits). It allocates nothing: no cudaMalloc, no cudaFree, no allocating library
 * call. Arguments, result and arithmetic are those of qgemm with path WOQ_PATH_BF16_TC.
 *   X, m, w, Y, stream  as for qgemm
 * Limit: m * k * 2 bytes (the bf16 copy of X, rounded up to 256) must not exceed 32 MiB,
 *   e.g. m <= 4096 at k = 4096; larger problems return WOQ_ESHAPE and queue nothing.
 * The first call on each device looks up the scratch array's device address (with that
 * device current) and caches it; make that first call before any stream capture.
 * All calls on a device share the scratch array. Each call overwrites the part it reads
 * before reading it, so nothing needs clearing, but two calls whose kernels overlap on the
 * GPU (e.g. on unordered streams) race on it: order them on one stream.
 * Errors: those of qgemm, with WOQ_ESHAPE also for the size limit.
 */
int qgemm_bf16_noalloc(const float *X, int64_t m, const woq_weight *w, float *Y, void *stream);

/*
 * woq_device_status -- synchronises the current device, then returns WOQ_ETIMEOUT if any
 * kernel of this library recorded a bounded wait that gave up since the last call with
 * clear != 0 (and clears the record if clear != 0), WOQ_ECUDA if synchronisation failed,
 * else WOQ_OK.
 */
int woq_device_status(int clear);

/*
 * woq_debug_set_wait_limit -- test hook for the bounded waits of the tensor-core qgemm kernel
 * and of qgemv_chain, applied to launches that follow. cycles > 0 sets the cycle budget of
 * every wait (qgemv_chain: of its waits for weights and for the other CTAs); in qgemv_chain,
 * cycles < 0 makes each CTA's waits for the other CTAs wait for one arrival more than there
 * are CTAs, bounded by -cycles cycles, so they give up deterministically;
 * 0 restores the default (2^32 cycles, about two seconds); cycles < 0 keeps the default
 * and makes the MMA-issuing thread of every CTA first wait on a barrier that nothing
 * arrives on, bounded by -cycles cycles, so the give-up path runs deterministically
 * without a hang (the kernel then records the event, drains, frees tensor memory and
 * returns; woq_device_status reports WOQ_ETIMEOUT). Process-wide host state; not
 * thread-safe against concurrent launches.
 */
void woq_debug_set_wait_limit(long long cycles);

/* Human-readable text for a status code (static storage; never NULL). */
const char *woq_status_str(int status);

/* Number of kernels this library has launched in this process (all devices). */
uint64_t woq_launch_count(void);

/* ABI version of this header: 1. */
int woq_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* WOQ_H */
