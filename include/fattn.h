/*
 * fattn.h -- C ABI of libfattn, a B200 (sm_100a) fused exact-attention library.
 *
 * Operation (forward).  For every batch b and head h, with Q, K, V each N x d
 * ("Q, K, V are all N x d", page 3, section 3 "从CUDA原理理解注意力机制的计算瓶颈"):
 *
 *     s_ij  = scale * <q_i, k_j>                  (scaled QK^T, page 2 "传统注意力为何容易受 IO 限制")
 *     s_ij  = -inf  where causal and j > i         (the mask of the same op chain; causal reading)
 *     P     = row softmax(s)                       (exact, page 2 "二、在线 Softmax 保持精确结果")
 *     O     = P V
 *     LSE_i = ln sum_j exp(s_ij)                   (the softmax statistic kept for the backward,
 *                                                   page 2 "三、融合算子减少中间张量落盘")
 *
 * computed as one fused, tiled kernel that never writes S or P to memory:
 * Q/K/V tiles stream through shared memory (page 1 "三、矩阵分块", page 2 "一、用分块计算提高
 * 片上数据复用"), the row max and row sum are kept online and earlier partial
 * outputs are rescaled when the max grows (page 3 "4.2 在线softmax技巧").
 *
 * Operation (backward).  Given dO = dL/dO, recompute S and P tile by tile from
 * Q, K and LSE (page 2 "四、反向传播选择重计算而非全量保存") and return
 *     dV = P^T dO,  dP = dO V^T,  dS = P o (dP - D),  D_i = sum_c dO_ic O_ic,
 *     dQ = scale * dS K,  dK = scale * dS^T Q.
 *
 * Tensor layout.  q, k, v, o, dout, dq, dk, dv are bfloat16, contiguous
 * [B, H, N, d] (d innermost, row stride d elements).  lse is float32 [B, H, N].
 * All pointers are DEVICE pointers on the current CUDA device and must be
 * 16-byte aligned.  Outputs must not alias inputs.
 *
 * Supported shapes: B, H, N >= 1 (any N); d in {32, 64, 96, 128} for the
 * forward and both backwards, and d = 256 for the forward and decoding only
 * (without dropout; the backward entry points return FATTN_ERR_UNSUPPORTED);
 * B * H * ceil(N / 128) * 128 < 2^31.  scale must be finite (any sign).  The
 * kernels work on 128-row tiles; a ragged last tile of each head is masked
 * (keys past N never receive weight, and rows past N are neither read nor
 * written).
 *
 * Ownership and asynchrony.  The caller allocates and owns every buffer,
 * including the backward workspace.  The library allocates no device memory at
 * run time.  Its only device state is static: 16 pairs of scheduling counters
 * for the causal forward, and the scratch array of fattn_bwd_noalloc.  It also
 * keeps 16 CUDA events per device, created by the first causal forward on that
 * device; these and the static arrays' device addresses are looked up once per
 * device, so the library must not be used across a reset of a device's context
 * (cudaDeviceReset, or the primary context released and created again).  Every
 * call only enqueues work on `stream` and returns; results are
 * valid once the stream has been synchronised.  Inputs must stay alive until
 * then.
 *
 * Errors.  Arguments are validated before anything is enqueued; an invalid
 * call returns a non-zero status and has no side effects.  A failed launch
 * returns FATTN_ERR_CUDA.  The library never synchronises the device and never
 * traps.  Kernels bound every wait on an on-chip barrier; a wait that runs out
 * (a library bug, never expected) records FATTN_ERR_DEVICE_TIMEOUT in a
 * per-device status word that fattn_device_status() reads.
 */
#ifndef FATTN_H_
#define FATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* fattn_stream_t; /* same object as cudaStream_t */

typedef enum {
  FATTN_OK = 0,
  FATTN_ERR_INVALID_ARG = 1,    /* null pointer, non-positive size, non-finite scale, too small workspace */
  FATTN_ERR_UNSUPPORTED = 2,    /* head dim not supported by this call, size overflow */
  FATTN_ERR_ALIGNMENT = 3,      /* a pointer is not 16-byte aligned */
  FATTN_ERR_CUDA = 4,           /* a CUDA runtime/driver call failed; see fattn_last_cuda_error() */
  FATTN_ERR_DEVICE_TIMEOUT = 5, /* a kernel's bounded wait ran out */
  FATTN_ERR_SCRATCH_TOO_SMALL = 6 /* fattn_bwd_noalloc: the shape needs more than its fixed scratch */
} fattn_status;

/*
 * Forward.  Writes o [B,H,N,d] (bf16) and lse [B,H,N] (fp32, natural log of
 * the row sum of exp of the scaled, masked scores).
 *   q, k, v : inputs, read only.
 *   causal  : 0 = no mask, 1 = query i attends keys 0..i.
 *   scale   : multiplies QK^T (usually 1/sqrt(d)).
 * One CTA per SM loops over units of two 128-row query tiles.  A causal launch
 * lets its CTAs claim units from one of the static counter pairs; the launch
 * that used the pair before has returned it to zero when it finished.  A pair
 * whose event (recorded after its previous launch) has completed is taken as it
 * is.  When every pair is busy, the launch takes the least recently handed-out
 * pair and makes `stream` wait on that pair's event first: nothing, if the
 * previous launch is earlier on the same stream, and otherwise an ordering
 * after that launch on its own stream.  A launch during stream capture assigns
 * units round-robin.  The schedule does not change the results: every unit is
 * computed the same way, whichever CTA takes it.
 */
int fattn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
              int B, int H, int N, int d, int causal, float scale,
              fattn_stream_t stream);

/*
 * General form of the forward.  Beyond fattn_fwd it takes
 *   - separate query and key lengths: q, o are [B, H, N_q, d], lse is [B, H, N_q];
 *     k, v are [B, H_kv, N_k, d];
 *   - grouped key/value heads: H must be a multiple of H_kv, and query head h of
 *     batch b reads key/value head h / (H / H_kv) of batch b (H_kv = H: one each;
 *     H_kv = 1: one for all);
 *   - a causal mask aligned at the bottom right: query i sees keys
 *     j <= i + N_k - N_q (the queries are the last N_q positions of the sequence).
 *     A query that sees no key (only when N_q > N_k) gets O = 0 and LSE = -inf;
 *   - dropout on the attention weights (page 2's op chain puts Dropout between the
 *     softmax and the product with V): each weight P_ij is kept with probability
 *     1 - dropout_p and then divided by 1 - dropout_p, or set to 0.  The draw for
 *     (flattened head b*H + h, query i, key j) is word j mod 4 of Philox4x32-10
 *     (Salmon et al., SC'11) at counter (i, floor(j / 4), b*H + h, offset) with key
 *     (seed mod 2^32, floor(seed / 2^32)); the weight is kept iff that word is
 *     >= floor(dropout_p * 2^32).  LSE is that of the undropped weights, and the
 *     backward regenerates the same mask from (seed, offset).
 * Constraints are fattn_fwd's, per length: B*H*ceil(N_q/128)*128 and
 * B*H_kv*ceil(N_k/128)*128 below 2^31; 0 <= dropout_p < 1.
 */
typedef struct fattn_fwd_params {
  const void* q;   /* [B, H, N_q, d] bf16 */
  const void* k;   /* [B, H_kv, N_k, d] bf16 */
  const void* v;   /* [B, H_kv, N_k, d] bf16 */
  void* o;         /* [B, H, N_q, d] bf16, written */
  float* lse;      /* [B, H, N_q] fp32, written */
  int B, H, H_kv, N_q, N_k, d;
  int causal;      /* 0 or 1 */
  float scale;
  float dropout_p; /* 0 = no dropout */
  unsigned long long seed;
  unsigned int offset;
} fattn_fwd_params;
int fattn_fwd_ex(const fattn_fwd_params* params, fattn_stream_t stream);

/*
 * Bytes of device workspace fattn_bwd needs for this shape (0 for an invalid
 * shape).  Layout inside (each part 256-byte aligned): D [B*H][Np] fp32 and
 * LSE*log2(e) [B*H][Np] fp32, where Np = ceil(N / 128) * 128 (each head padded
 * to whole 128-row tiles, padding rows 0), then the fp32 dQ accumulator
 * [B,H,N,d].
 */
size_t fattn_bwd_workspace_size(int B, int H, int N, int d);

/*
 * Backward.  Inputs q, k, v, o (the forward output), dout (dL/dO) and lse (the
 * forward statistic) are read only.  Writes dq, dk, dv (bf16, [B,H,N,d]).
 * workspace: device memory of at least fattn_bwd_workspace_size() bytes,
 * 256-byte aligned, owned by the caller; its contents on entry do not matter.
 * Deterministic up to the order of fp32 additions into the dQ accumulator.
 */
int fattn_bwd(const void* q, const void* k, const void* v, const void* o,
              const void* dout, const float* lse, void* dq, void* dk, void* dv,
              int B, int H, int N, int d, int causal, float scale,
              void* workspace, size_t workspace_bytes, fattn_stream_t stream);

/*
 * General form of the backward, for the forward of fattn_fwd_ex: the same
 * shapes, mask, grouping and dropout arguments (seed and offset must be those of
 * the forward), plus
 *   dout [B, H, N_q, d]; dq [B, H, N_q, d]; dk, dv [B, H_kv, N_k, d] (a shared
 *   key/value head gets the sum over the query heads of its group);
 *   deterministic: 0 = dQ accumulated with fp32 reduce-adds as in fattn_bwd
 *     (reproducible only up to the order of those additions); 1 = dQ computed
 *     by a separate pass that owns each query tile and recomputes S and dP for
 *     it, so that every output is bit-identical from run to run;
 *   workspace: device memory of at least fattn_bwd_ex_workspace_size(params)
 *     bytes, 256-byte aligned (the deterministic backward needs no accumulator).
 */
typedef struct fattn_bwd_params {
  const void* q;
  const void* k;
  const void* v;
  const void* o;      /* the forward's output */
  const void* dout;   /* dL/dO */
  const float* lse;   /* the forward's statistic */
  void* dq;
  void* dk;
  void* dv;
  int B, H, H_kv, N_q, N_k, d;
  int causal;
  float scale;
  float dropout_p;
  unsigned long long seed;
  unsigned int offset;
  int deterministic;
  void* workspace;
  size_t workspace_bytes;
} fattn_bwd_params;
size_t fattn_bwd_ex_workspace_size(const fattn_bwd_params* params);
int fattn_bwd_ex(const fattn_bwd_params* params, fattn_stream_t stream);

/*
 * Attention for incremental decoding: a few new query rows per sequence against
 * a long key/value cache.  The result is that of fattn_fwd_ex (without dropout);
 * the work is laid out for this shape instead: the G = H / H_kv query heads that
 * share a key/value head are packed into one 128-row tile (G * N_q rows; more
 * rows take more tiles), and the keys of each (key/value head, row tile) are
 * split into num_splits ranges processed by separate CTAs, whose partial outputs
 * a second kernel merges by their log-sum-exp.  Page 2 ("落地使用时应关注什么")
 * separates this incremental inference, bound by reading the cache, from
 * training.
 *   q  [B, H, N_q, d] bf16; o [B, H, N_q, d] bf16 and lse [B, H, N_q] fp32, written.
 *   k, v: the cache, [B, H_kv, N_k_cap, d] bf16 with N_k_cap >= N_k; only the
 *     first N_k rows of each head are read.
 *   causal: 1 = query i sees keys j <= i + N_k - N_q (the new rows are the last
 *     N_q positions of the sequence).
 *   num_splits: key ranges per (key/value head, row tile); 0 lets the library
 *     choose (about four CTAs per SM in all); values above ceil(N_k / 128) are
 *     reduced to it.
 *   workspace: fattn_decode_workspace_size(params) bytes (0 when one split is
 *     used), 256-byte aligned; may be null when that size is 0.
 */
typedef struct fattn_decode_params {
  const void* q;
  const void* k;
  const void* v;
  void* o;
  float* lse;
  int B, H, H_kv, N_q, N_k, N_k_cap, d;
  int causal;
  float scale;
  int num_splits;
  void* workspace;
  size_t workspace_bytes;
} fattn_decode_params;
size_t fattn_decode_workspace_size(const fattn_decode_params* params);
int fattn_decode(const fattn_decode_params* params, fattn_stream_t stream);

/*
 * Backward that allocates nothing and takes no workspace argument.
 *
 * The pages the library follows have no counterpart of this call.  It is for
 * callers that cannot allocate device memory or hand over a buffer of their
 * own: for example a plugin running inside a host application that owns all
 * device memory and gives the plugin no allocator, or a serving loop that
 * reserves its memory once at start-up and forbids allocations (and the
 * device-wide synchronisation an allocation can cause) on its request path.
 *
 * Arguments, layout, results and errors are those of fattn_bwd without the
 * workspace.  The scratch space fattn_bwd takes from its workspace comes
 * instead from one fixed array of FATTN_NOALLOC_SCRATCH_BYTES bytes (32 MiB)
 * that the library keeps in device memory; every GPU that loads the library
 * holds that array until the process exits.  A shape is accepted exactly when
 * fattn_bwd_workspace_size(B, H, N, d) <= FATTN_NOALLOC_SCRATCH_BYTES; larger
 * ones are rejected with FATTN_ERR_SCRATCH_TOO_SMALL before anything is
 * enqueued.  For N a multiple of 128 that means B*H*N <= 64512 at d = 128 and
 * B*H*N <= 126976 at d = 64; for other N the per-head statistics are padded to
 * whole 128-row tiles and count too, so the limit on B*H*N is lower.
 *
 * The first call on a device looks up the array's device address and caches
 * it; make that first call before any stream capture on that device.  The
 * cached address belongs to the device's current context: the library must not
 * be used across a reset of that context (cudaDeviceReset, or the primary
 * context released and created again), which would leave it stale.  All calls
 * on one device share the array, and each call re-initialises what must start
 * at zero, so calls whose executions overlap on the GPU (on different streams,
 * or from several host threads) race on it and must be serialised by the caller.
 */
#define FATTN_NOALLOC_SCRATCH_BYTES (32u << 20)
int fattn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                      const void* dout, const float* lse, void* dq, void* dk, void* dv,
                      int B, int H, int N, int d, int causal, float scale,
                      fattn_stream_t stream);

/*
 * The three stages fattn_bwd runs, exposed so that callers can schedule or time
 * them separately.  They must run in this order on one stream with the same
 * shape, scale and workspace; fattn_bwd(...) is exactly
 *   fattn_bwd_preprocess; fattn_bwd_dkdv; fattn_bwd_dq.
 *
 * fattn_bwd_preprocess: D_i = sum_c dout_ic o_ic and LSE_i*log2(e) into the
 *   workspace, and zeroes the workspace's fp32 dQ accumulator.
 * fattn_bwd_dkdv: writes dk, dv and adds dS K (unscaled) into the accumulator.
 *   Reads q, k, v, dout and the preprocess results.
 * fattn_bwd_dq: dq = bf16(scale * accumulator).
 * Validation and errors are those of fattn_bwd.
 */
int fattn_bwd_preprocess(const void* o, const void* dout, const float* lse, int B, int H, int N, int d,
                         void* workspace, size_t workspace_bytes, fattn_stream_t stream);
int fattn_bwd_dkdv(const void* q, const void* k, const void* v, const void* dout, void* dk, void* dv,
                   int B, int H, int N, int d, int causal, float scale,
                   void* workspace, size_t workspace_bytes, fattn_stream_t stream);
int fattn_bwd_dq(void* dq, int B, int H, int N, int d, float scale,
                 void* workspace, size_t workspace_bytes, fattn_stream_t stream);

/* Static, human-readable text for a status code. */
const char* fattn_status_string(int status);

/* Text of the last CUDA error seen by this thread inside the library ("" if none). */
const char* fattn_last_cuda_error(void);

/*
 * Reads (synchronously) the current device's kernel status word: FATTN_OK, or
 * FATTN_ERR_DEVICE_TIMEOUT if some kernel's bounded wait ran out since the last
 * clear.  clear != 0 resets the word.  Returns FATTN_ERR_CUDA if the read fails.
 */
int fattn_device_status(int clear);

/*
 * Failure-detection self-test: enqueues one small kernel whose single warp waits on
 * an on-chip barrier that nothing completes, with the same bounded wait the
 * attention kernels use.  After about one second the wait gives up, records its
 * site in the device status word and the kernel returns; no fault, trap or hang is
 * involved, and the context stays usable.  A following fattn_device_status()
 * reports FATTN_ERR_DEVICE_TIMEOUT (and clears it if asked).  Lets a caller, or a
 * test, check that timeouts are detected and reported on its device.
 */
int fattn_selftest_wait_timeout(fattn_stream_t stream);

/* Library version, e.g. 0x000200 for 0.2.0. */
int fattn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FATTN_H_ */
