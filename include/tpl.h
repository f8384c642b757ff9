/*
 * tpl.h -- C ABI of the tensor-parallel sharded-linear library for B200 (sm_100a).
 *
 * One GPU computes every tensor-parallel (TP) shard of a transformer block's
 * linear layers locally; the last group of calls splits the same linears over
 * GPUs, one process per GPU.  The calls follow the shapes of the pages they
 * come from:
 *
 *   - nanotron rules, "Tensor-Parallel Component Patterns" (sections
 *     "Attention Module" and "MLP Module"): TP linears take the full logical
 *     dimensions plus the TP size and shard internally; c_fc is column-parallel
 *     with intermediate/tp columns per rank, then GELU, then the row-parallel
 *     c_proj.  Hidden states arrive as [batch, seq, hidden]; this ABI takes the
 *     flattened row count M = batch * seq.
 *   - DeepSpeed "Class SubParamLinearLayer": a fused weight made of several
 *     logical sub-parameters (fused QKV, unequal GQA widths) partitioned one
 *     by one along the output dim; forward is matmul(input, W^T) + bias; the
 *     bias must match the output size.
 *   - google-research two_d_parallel_xmap.py: allgather_layernorm (RMSNorm,
 *     epsilon inside the rsqrt, optional centred scale), the o_wo section
 *     (per-shard partial products summed over the sharded contraction) and
 *     the residual section; unembed_manual (fp32 logits).
 *   - Tenstorrent lm_head_1d.py: vocab-sharded, chunked LM head
 *     (LMHead1D.from_model_args split sizes); the argmax over shards, left to
 *     the caller there, is fused on the device here.
 *
 * Conventions for every call:
 *   - Pointers marked "device" are CUDA device pointers owned by the caller;
 *     the library never frees or keeps them.  Pointers marked "host" are read
 *     during the call only.
 *   - Matrices are dense and row-major; weights use the nn.Linear layout
 *     [out][in], so both GEMM operands are K-contiguous.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Device
 *     work is enqueued on it and the call returns without waiting.  Argument
 *     checks happen on the host before anything is enqueued; a rejected call
 *     enqueues nothing.
 *   - bf16 in -> bf16 out with fp32 accumulation and fp32 epilogue maths;
 *     fp32 in -> fp32 out.
 *   - A kernel that gives up waiting on its own pipeline records
 *     TPL_ERR_TIMEOUT in a per-device status word; tpl_get_device_status reads
 *     and clears it.
 *   - The library allocates no device memory.  Its only device state is three
 *     module-level variables per device, loaded with the library: the status
 *     word, the fixed scratch of tpl_lmhead_argmax_static and the pointer to
 *     an optional trace buffer (tpl_trace_set).  The calls are thread-safe.
 *   - Environment variables (for measurements; results are the same under
 *     every setting): TPL_PDL=0 launches without programmatic dependent
 *     launch; TPL_GEMM_CTA_PAIRS=0 keeps every GEMM on single CTAs;
 *     TPL_GEMM_GROUP_M and TPL_GEMM_KSERP set the CTA-pair GEMM's tile raster
 *     (m-blocks per group, K order reversed on alternate tiles); TPL_LMHEAD_TN
 *     picks the decode LM-head kernel for batches of up to 32 rows (2, the
 *     default: the batch as a 64-row MMA operand; 1: a 128-row one; 0: the
 *     swap-AB kernel that larger batches use) and TPL_LMHEAD_RANGES=0 gives
 *     the transposed kernel uniform vocab slabs instead of one contiguous
 *     range per CTA.  TPL_PDL and TPL_LMHEAD_TN are read once per process,
 *     the others per call.
 */
#ifndef TPL_H
#define TPL_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TPL_OK = 0,
  TPL_ERR_NULL = 1,         /* a required pointer is NULL                          */
  TPL_ERR_SHAPE = 2,        /* a size is out of range or sizes disagree            */
  TPL_ERR_INDIVISIBLE = 3,  /* a partition leaves a rank without rows, or a size
                               is not a multiple of the alignment unit             */
  TPL_ERR_DTYPE = 4,        /* unknown dtype or activation                         */
  TPL_ERR_ALIGN = 5,        /* a pointer or row stride breaks the 16-byte rule     */
  TPL_ERR_CUDA = 6,         /* a CUDA runtime/driver call failed                   */
  TPL_ERR_TIMEOUT = 7,      /* a kernel gave up waiting on its pipeline            */
  TPL_ERR_UNSUPPORTED = 8   /* valid request outside what this library implements  */
} tpl_status;

typedef enum { TPL_FP32 = 0, TPL_BF16 = 1 } tpl_dtype;

typedef enum {
  TPL_ACT_NONE = 0,
  TPL_ACT_GELU_ERF = 1,   /* 0.5 y (1 + erf(y / sqrt 2))                           */
  TPL_ACT_GELU_TANH = 2   /* 0.5 y (1 + tanh(sqrt(2/pi) (y + 0.044715 y^3)))       */
} tpl_act;

#define TPL_MAX_TP 64
#define TPL_MAX_SUB 8

/*
 * Per-rank layout of a column-parallel fused weight (caller-owned POD).
 * For rank r and sub-parameter j: rows src_off[r][j] .. + width[r][j] of the
 * fused weight (and the same entries of the fused bias) produce columns
 * dst_off[r][j] .. of rank r's shard.  shard_base[r] is the sum of the shard
 * widths of the lower ranks.
 */
typedef struct {
  int32_t tp_size;
  int32_t n_sub;
  int64_t logical_out;
  int64_t width[TPL_MAX_TP][TPL_MAX_SUB];
  int64_t src_off[TPL_MAX_TP][TPL_MAX_SUB];
  int64_t dst_off[TPL_MAX_TP][TPL_MAX_SUB];
  int64_t shard_width[TPL_MAX_TP];
  int64_t shard_base[TPL_MAX_TP];
} tpl_partition;

/*
 * Sub-parameter partition (DeepSpeed "Class SubParamLinearLayer": the shape
 * spec (n, -1) / ((q, k, v), -1) with partition_dim 0; nanotron "MLP Module":
 * intermediate // tp columns per rank).  Host only, no device work.
 *
 *   sub_sizes  host, [n_sub] logical output sizes in the fused order (q, k, v).
 *   n_sub      1 .. TPL_MAX_SUB.     tp_size  1 .. TPL_MAX_TP.
 *   align      rows per indivisible unit (head_dim for attention, 1 for MLP).
 *   out        host, filled on success; untouched on error.
 *
 * Each sub-parameter is cut into sub_sizes[j] / align units; rank r gets
 * units / tp + (r < units % tp) of them.  Errors: TPL_ERR_NULL,
 * TPL_ERR_SHAPE (counts or sizes out of range), TPL_ERR_INDIVISIBLE (size not
 * a multiple of align, or a rank left with zero rows of some sub-parameter).
 */
tpl_status tpl_partition_subparams(const int64_t* sub_sizes, int32_t n_sub, int32_t tp_size,
                                   int64_t align, tpl_partition* out);

/*
 * Column-parallel linear with sub-parameter partitioning, bias and activation
 * fused in the epilogue (SubParamLinearLayer.forward; nanotron c_fc + F.gelu).
 *
 *   p      host, a partition from tpl_partition_subparams.
 *   x      device, [M][K] activations (dtype dt).
 *   w      device, [p->logical_out][K] fused weight, nn.Linear layout.
 *   bias   device, [p->logical_out] in the fused order, or NULL.
 *   y      device; rank r's shard is the row-major [M][shard_width[r]] block
 *          starting at element M * shard_base[r].
 *   Y_r = act(X W_r^T + b_r).  M == 0 is a no-op (x, w, y may then be NULL).
 *
 * bf16 runs on the tcgen05 tensor cores and needs K % 8 == 0 and 16-byte
 * aligned x and w (else TPL_ERR_ALIGN); fp32 runs on the CUDA cores.
 */
tpl_status tpl_column_linear(const tpl_partition* p, const void* x, int64_t M, int64_t K,
                             const void* w, const void* bias, tpl_dtype dt, tpl_act act,
                             void* y, void* stream);

/*
 * Row-parallel linear whose per-shard partial products are reduced on the
 * device inside the GEMM (google-research o_wo section; nanotron c_proj):
 *   Y = sum_{r=0}^{tp-1} H_r W2_r^T (+ bias) (+ residual)
 * The shards are consecutive stretches of one fp32 accumulator, so the sum is
 * taken in rank order with no extra pass.
 *
 *   h         device; rank r's block [M][k_w[r]] starts at element
 *             M * sum_{q<r} k_w[q] (the layout tpl_column_linear writes).
 *   k_w       host, [tp] contraction width of each rank.
 *   w         device; rank r's block [N][k_w[r]] starts at element
 *             N * sum_{q<r} k_w[q] (columns of the unsharded [N][K] weight).
 *   bias      device [N] or NULL, added once after the sum.
 *   residual  device [M][N] or NULL; may alias y (x <- x + f(x)).
 *   y         device [M][N].
 *   partials  device [tp][M][N] fp32 or NULL.  When given, each rank's
 *             partial product is also written out unreduced (a check of the
 *             reduction; slower: one extra pass per rank).
 *   M == 0 is a no-op (h, w, y may then be NULL).
 *
 * bf16 needs every k_w[r] % 8 == 0 and 16-byte aligned h and w.  The bf16
 * kernel takes at most two contraction widths, each held by a contiguous run
 * of ranks (k_w = {a, .., a, b, .., b}, the shape tpl_partition_subparams
 * gives an uneven split); other patterns return TPL_ERR_UNSUPPORTED.  fp32
 * takes any widths.
 */
tpl_status tpl_row_linear_reduce(const void* h, const int64_t* k_w, int32_t tp, int64_t M,
                                 int64_t N, const void* w, const void* bias,
                                 const void* residual, tpl_dtype dt, void* y, float* partials,
                                 void* stream);


/*
 * Column-parallel linear of RMSNorm(x) with the norm fused into the GEMM
 * (google-research allgather_layernorm; nanotron "MLP Module": RMSNorm, then
 * c_fc).  Since RMSNorm(x) W^T = diag(rsqrt(mean(x^2) + eps)) x (W diag(g))^T,
 * the norm's scale g is folded into the weight once (tpl_fold_norm_scale) and
 * the per-row factor is applied in the GEMM epilogue:
 *   Y_r = act(rsqrt(mean_k x[m][k]^2 + eps) * (x W'_r^T)[m] + b_r)
 * The GEMM's CTAs compute every row's factor from x (fp32 sums of the bf16
 * values) while their first tiles' MMAs run, so no normalised copy of x is
 * written or read.  Rounding: x enters the GEMM unnormalised and g is rounded
 * into W' once, where the unfused path rounds the normalised x to bf16.
 *
 *   x          device bf16 [M][K], the raw activations.
 *   w          device bf16 [p->logical_out][K], the weight with g folded in.
 *   bias, act, y, p   as tpl_column_linear.   eps >= 0.
 *   workspace  device, tpl_column_linear_rmsnorm_workspace_size(M) bytes
 *              (the per-row factors and their ready flags), 256-byte aligned,
 *              ZERO-FILLED before its first use, reusable without clearing
 *              (each call stamps its flags with a value fresh to that call).
 *              Calls whose work overlaps on the GPU must not share one.
 * bf16 only (K % 8 == 0, 16-byte aligned x and w).  Errors as
 * tpl_column_linear, plus TPL_ERR_SHAPE for a short workspace.
 */
tpl_status tpl_column_linear_rmsnorm_workspace_size(int64_t M, size_t* bytes);

tpl_status tpl_column_linear_rmsnorm(const tpl_partition* p, const void* x, int64_t M, int64_t K,
                                     const void* w, const void* bias, float eps, tpl_act act,
                                     void* y, void* workspace, size_t ws_bytes, void* stream);

/*
 * Folds an RMSNorm scale into the columns of the weight that follows it:
 *   w_out[n][k] = bf16(w[n][k] * g[k]),  g = 1 + scale (centered) or scale
 * (google-research allgather_layernorm: scale += 1.0 when centring).  A
 * one-time weight transformation for tpl_column_linear_rmsnorm.
 *
 *   w      device bf16 [rows][K].   scale  device fp32 [K].
 *   w_out  device bf16 [rows][K]; may alias w.
 * Requirements: K % 8 == 0; w, w_out and scale 16-byte aligned (else
 * TPL_ERR_ALIGN).  rows == 0 is a no-op.
 */
tpl_status tpl_fold_norm_scale(const void* w, int64_t rows, int64_t K, const float* scale,
                               int32_t centered, void* w_out, void* stream);

/*
 * RMSNorm (google-research allgather_layernorm; weight-gathered layernorm):
 *   y = x / sqrt(mean(x^2) + eps) * g,  g = 1 + scale (centered != 0),
 *   g = scale (centered == 0), or g = 1 (scale == NULL).
 * fp32 maths, one rounding on store.
 *
 *   x      device [M][H];  y  device [M][H], may alias x.
 *   scale  device fp32 [H] or NULL.
 *   M == 0 is a no-op (x, y may then be NULL).
 */
tpl_status tpl_rmsnorm(const void* x, int64_t M, int64_t H, const float* scale, int32_t centered,
                       float eps, tpl_dtype dt, void* y, void* stream);

/*
 * Sequence parallelism around the TP linears (nanotron "MLP Module": the
 * row-parallel c_proj hands rank r the rows [batch, seq // tp, hidden]).
 * Activations of a sequence-parallel region are stored rank-major: rank r's
 * slice [batch][seq/tp][*] (tokens r*seq/tp .. (r+1)*seq/tp of every sequence)
 * starts at row r*batch*(seq/tp).  On one GPU the reduce-scatter and the
 * all-gather are row remaps inside the GEMMs; no data moves twice.
 *
 * tpl_row_linear_reduce_scatter: as tpl_row_linear_reduce with M = batch*seq,
 * but y (and residual, if given) are in the rank-major layout, so rank r's
 * slice holds the summed output of its tokens.  seq % tp != 0 ->
 * TPL_ERR_INDIVISIBLE.
 */
tpl_status tpl_row_linear_reduce_scatter(const void* h, const int64_t* k_w, int32_t tp,
                                         int64_t batch, int64_t seq, int64_t N, const void* w,
                                         const void* bias, const void* residual, tpl_dtype dt,
                                         void* y, void* stream);

/*
 * tpl_column_linear_allgather: as tpl_column_linear with M = batch*seq, but x
 * is read from the rank-major layout (the all-gather along the sequence that
 * precedes a column-parallel linear), tp = p->tp_size.  The bf16 path needs
 * (seq/tp) % 128 == 0 (else TPL_ERR_UNSUPPORTED).
 */
tpl_status tpl_column_linear_allgather(const tpl_partition* p, const void* x, int64_t batch,
                                       int64_t seq, int64_t K, const void* w, const void* bias,
                                       tpl_dtype dt, tpl_act act, void* y, void* stream);

/*
 * Column-parallel fused SwiGLU projection (google-research, "SwiGLU" section
 * and the fused q_wi projection: swish(wi0) * wi1).
 *
 *   x   device bf16 [M][K].
 *   w   device bf16 [2F][K]: the F rows of wi0, then the F rows of wi1.
 *   h   device bf16; rank r's block [M][F_r] starts at element M*sum_{q<r} F_q,
 *       F_r = F/tp + (r < F%tp); h_r = silu(X wi0_r^T) * (X wi1_r^T),
 *       silu(a) = a / (1 + exp(-a)).
 * Each 256-wide tile pairs a 128-column block of wi0 with the same block of
 * wi1, so the gate is applied in the epilogue.  bf16 only (fp32 ->
 * TPL_ERR_UNSUPPORTED); F < tp -> TPL_ERR_INDIVISIBLE.
 */
tpl_status tpl_swiglu_column_linear(const void* x, int64_t M, int64_t K, const void* w, int64_t F,
                                    int32_t tp, tpl_dtype dt, void* h, void* stream);

/*
 * Vocab-sharded embedding lookup (google-research embed_manual, 'embed'
 * scope): rank r holds table rows r*shard .. (r+1)*shard (shard = ceil(V/tp)),
 * keeps its row where 0 <= id - r*shard < its row count, and the embedding is
 * the sum over ranks (fp32, one rounding).  Ids outside [0, V) give zeros.
 *
 *   ids    device int32 [n].     table  device [V][H] (dtype dt).
 *   out    device [n][H].        n == 0 is a no-op.
 */
tpl_status tpl_embedding_lookup(const int32_t* ids, int64_t n, const void* table, int64_t V,
                                int64_t H, int32_t tp, tpl_dtype dt, void* out, void* stream);

/*
 * Bytes of device workspace tpl_lmhead_argmax needs for B rows and tp shards.
 * Errors as for tpl_lmhead_argmax's shape checks.
 */
tpl_status tpl_lmhead_workspace_size(int64_t B, int64_t V, int32_t tp, int32_t n_chunks,
                                     size_t* bytes);

/*
 * Decode LM head over a vocab split into tp shards of n_chunks chunks
 * (Tenstorrent LMHead1D; google-research unembed_manual), with the per-shard
 * and the global argmax fused in.
 *
 * Layout (LMHead1D.from_model_args with tile 1): shard = ceil(V / tp);
 * chunk_cols = ceil(shard / n_chunks); split sizes [chunk_cols] * (n - 1) +
 * [shard - sum]; the call is rejected (TPL_ERR_SHAPE) unless that gives exactly
 * n_chunks splits with a positive last one.  Column j of chunk c on shard r
 * is global id r * shard + sum(split[:c]) + j; ids >= V are padding and never
 * reported.
 *
 *   x          device bf16 [B][K], 1 <= B <= 256, K % 8 == 0.
 *   w          device bf16 [V][K].
 *   logits     device fp32 [B][V] or NULL (logits[b][v] = x[b] . w[v]).
 *   shard_max  device fp32 [tp][B]; -inf for a shard with no real id.
 *   shard_idx  device int32 [tp][B] global ids; -1 for an empty shard.
 *   ids        device int32 [B] global argmax.
 *   workspace  device, ws_bytes >= tpl_lmhead_workspace_size(...), 16-byte
 *              aligned.  It must be zero-filled before its first use; every
 *              call that completes leaves it zero-filled again, so it can be
 *              reused without clearing.  After TPL_ERR_TIMEOUT, clear it again.
 * Ties go to the lowest global id.  Calls sharing a workspace must not overlap.
 */
tpl_status tpl_lmhead_argmax(const void* x, int64_t B, int64_t K, const void* w, int64_t V,
                             int32_t tp, int32_t n_chunks, float* logits, float* shard_max,
                             int32_t* shard_idx, int32_t* ids, void* workspace, size_t ws_bytes,
                             void* stream);

/*
 * tpl_lmhead_argmax with no workspace argument, for callers that cannot
 * allocate device memory.  (No counterpart on the pages: this is an
 * integration entry point of this library.)  Some callers cannot call
 * cudaMalloc: a plugin inside a host framework that owns all device memory
 * and hands the plugin only its input and output buffers, or a
 * latency-critical decode loop where an allocation (which can synchronise the
 * device) is not allowed.  This entry point allocates nothing: its scratch
 * (per-shard keys and a completion counter) lives in a fixed array of
 * TPL_LMHEAD_STATIC_SCRATCH_BYTES bytes inside the library, which every GPU
 * that loads the library holds until the process exits.
 *
 * Arguments, layout, outputs and ties are as for tpl_lmhead_argmax; the
 * caller still passes x, w and every output buffer.
 *   - Sizes whose scratch (tp * B * 8 + 16 bytes, rounded up to 256) exceeds
 *     TPL_LMHEAD_STATIC_SCRATCH_BYTES are rejected with TPL_ERR_SHAPE.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture on the device.  The address is kept for the
 *     device's CUDA context: after cudaDeviceReset the next call looks it up
 *     again in the new context (so again outside any stream capture), and
 *     the array starts over at zero.
 *   - Every check of tpl_lmhead_argmax runs before anything is enqueued: a
 *     rejected call enqueues nothing, not even the clear below.
 *   - Every call on a device shares the one array and clears the part it uses
 *     (cudaMemsetAsync on `stream`) before the kernel.  Calls whose work
 *     overlaps on the GPU (different streams, or different host threads)
 *     race on it: order them on one stream.
 */
#define TPL_LMHEAD_STATIC_SCRATCH_BYTES 65536

tpl_status tpl_lmhead_argmax_static(const void* x, int64_t B, int64_t K, const void* w, int64_t V,
                                    int32_t tp, int32_t n_chunks, float* logits, float* shard_max,
                                    int32_t* shard_idx, int32_t* ids, void* stream);

/* ------------------------------------------------------------------------
 * The TP linears split over GPUs: one process per GPU, rank `rank` of `tp`.
 * ------------------------------------------------------------------------ */

#define TPL_MAX_GATHER 16

/*
 * This rank's shard of a column-parallel linear over the all-gathered tokens
 * (nanotron "MLP Module": the sequence-parallel activations [batch, seq // tp,
 * hidden] of every rank are gathered ahead of the column-parallel c_fc; DeepSpeed
 * "Class SubParamLinearLayer" for the shard's pieces).  Computes, for all
 * batch * seq tokens,  Y = act(X W^T + b)  with this rank's weight rows, where
 * the GEMM reads each 128-row tile of X straight from the rank that owns those
 * tokens, so the all-gather overlaps the GEMM tile by tile.
 *
 *   p       partition of this rank's weight (tp_size 1 for a plain shard; the
 *           shard's fused pieces, e.g. q, k, v, as sub-parameters).
 *   peer_x  HOST array of tp device pointers: peer_x[q] is rank q's token slice,
 *           bf16 [batch][seq / tp][K] (tokens q * seq/tp .. of every sequence);
 *           a mapping of that GPU's buffer for q != this rank.  Read with plain
 *           TMA loads.
 *   w, bias, act, y  as tpl_column_linear with M = batch * seq (y holds every
 *           token's row of this rank's shard).
 * Requirements: tp <= TPL_MAX_GATHER and (seq / tp) % 128 == 0 (else
 * TPL_ERR_UNSUPPORTED), seq % tp == 0 (else TPL_ERR_INDIVISIBLE), K % 8 == 0
 * and 16-byte aligned slices and w (else TPL_ERR_ALIGN).  bf16 only.
 * Completion: every rank's slice must be complete before this call's work on
 * `stream` starts (a stream-ordered collective after the producers on every
 * rank), and must not be overwritten until this call's work has completed.
 */
tpl_status tpl_column_linear_gather(const tpl_partition* p, void* const* peer_x, int32_t tp,
                                    int64_t batch, int64_t seq, int64_t K, const void* w,
                                    const void* bias, tpl_act act, void* y, void* stream);

/*
 * This rank's shard of a row-parallel linear whose reduction is a
 * reduce-scatter over the token dimension (google-research: each shard's
 * "{YZ unreduced}" partial, reduced afterwards; nanotron "MLP Module": the
 * c_proj output is [batch, seq // tp, hidden] per rank).  The partial
 *   P = H_rank W_rank^T   (bf16 in, fp32 accumulate, stored bf16)
 * is written by the GEMM epilogue straight into the receive buffer of the rank
 * that owns each token, so the exchange overlaps the GEMM tile by tile.
 *
 *   h     device bf16 [batch * seq][K], this rank's contraction slice of the
 *         activations (token b * seq + t in row b * seq + t).
 *   w     device bf16 [N][K], this rank's columns of the unsharded [N][tp*K]
 *         weight.
 *   peer  HOST array of tp device pointers: peer[q] is rank q's receive buffer,
 *         bf16 [tp][batch][seq / tp][N] (slot s holds rank s's partial of the
 *         tokens q * seq/tp .. (q+1) * seq/tp - 1 of every sequence).  For
 *         q != rank it must be a mapping of that GPU's buffer into this process
 *         (CUDA IPC or equivalent); the kernel writes it with plain stores.
 *         Token t of sequence b goes to peer[t / (seq/tp)], slot `rank`, row
 *         b * seq/tp + t % (seq/tp).
 * Requirements: seq % tp == 0 (else TPL_ERR_INDIVISIBLE), K % 8 == 0, h and w
 * 16-byte aligned (else TPL_ERR_ALIGN), batch * seq <= INT32_MAX.
 * Completion: the writes are complete when this call's work on `stream` is;
 * a rank may read its receive buffer only after every rank's scatter has
 * completed (a stream-ordered collective, e.g. an all-reduce of one element,
 * after the scatter on every rank).
 */
tpl_status tpl_row_linear_scatter(const void* h, int64_t K, int64_t batch, int64_t seq, int64_t N,
                                  const void* w, int32_t rank, int32_t tp, void* const* peer,
                                  void* stream);


/*
 * The reduction step of the reduce-scatter above, on the rank that owns a
 * token slice:  y[i][n] = bf16( sum_{s < tp} recv[s][i][n] + bias[n]
 * + residual[i][n] ), summed in fp32 in rank order (the order of the one-GPU
 * tpl_row_linear_reduce).
 *   recv      device bf16 [tp][rows][N] (the receive buffer, rows = batch*seq/tp).
 *   bias      device bf16 [N] or NULL.   residual  device bf16 [rows][N] or NULL.
 *   y         device bf16 [rows][N]; may alias residual.
 * rows == 0 is a no-op.  TPL_ERR_SHAPE if tp is outside [1, TPL_MAX_TP], N is
 * outside [1, INT32_MAX], rows < 0, or tp * rows * N overflows int64_t.
 */
tpl_status tpl_reduce_slots(const void* recv, int32_t tp, int64_t rows, int64_t N,
                            const void* bias, const void* residual, void* y, void* stream);

/*
 * tpl_reduce_slots and the RMSNorm of its result in one pass (google-research
 * allgather_layernorm applied to the next layer's input): the residual stream
 * and the next layer's normalised input come out of one read of the slots, so
 * the next layer needs no RMSNorm launch of its own.
 *   y[i][n]  = bf16( sum_{s < tp} recv[s][i][n] + bias[n] + residual[i][n] ),
 *              exactly as tpl_reduce_slots;
 *   xn[i][n] = bf16( y[i][n] * rsqrt(mean_n y[i][n]^2 + eps) * g[n] ), on the
 *              bf16 values of y, g = 1 + scale (centered), scale, or 1 (scale
 *              NULL), in fp32 as tpl_rmsnorm (the sum of squares in another
 *              order, so the last bit of an element can differ).
 *   recv, bias, residual, y  as tpl_reduce_slots (y may alias residual).
 *   scale     device fp32 [N] or NULL.   xn  device bf16 [rows][N]; aliases
 *             none of the other buffers.
 * rows == 0 is a no-op.  Errors: as tpl_reduce_slots, plus TPL_ERR_SHAPE for
 * eps < 0 or NaN, TPL_ERR_NULL for a NULL xn, TPL_ERR_ALIGN unless N % 8 == 0
 * and every buffer is 16-byte aligned, TPL_ERR_UNSUPPORTED for N > 16384.
 */
tpl_status tpl_reduce_slots_rmsnorm(const void* recv, int32_t tp, int64_t rows, int64_t N,
                                    const void* bias, const void* residual, void* y,
                                    const float* scale, int32_t centered, float eps, void* xn,
                                    void* stream);

/*
 * The same reduction, with the slice stored into EVERY rank's full output
 * (google-research: the row-parallel partials reduced over the sharded
 * contraction axis; nanotron "MLP Module" without sequence parallelism, where
 * each rank keeps the whole [batch, seq, hidden] output).  Rank `rank` owns
 * tokens rank * seq/tp .. (rank + 1) * seq/tp of every sequence; it computes
 *   S[b][t][n] = bf16( sum_{s < tp} recv[s][b][t][n] + bias[n]
 *                      + residual[b * seq + rank * seq/tp + t][n] )
 * and stores S at row b * seq + rank * seq/tp + t of peer_y[q] for every q.
 * After tpl_row_linear_scatter, a barrier and this call on every rank, and a
 * second barrier, every rank's output holds the full
 *   Y = sum_r H_r W2_r^T (+ bias) (+ residual):
 * an all-reduce whose data moves only in the GEMM epilogue's and this
 * kernel's peer stores.
 *   recv      device bf16 [tp][batch][seq/tp][N], this rank's receive buffer.
 *   bias      device bf16 [N] or NULL.
 *   residual  device bf16 [batch * seq][N] or NULL: this rank's own copy of
 *             the residual stream (identical on every rank); it may alias
 *             peer_y[rank] (in place), as each element of this rank's token
 *             rows is read and then stored by one thread, and no other rank
 *             writes those rows.
 *   peer_y    array of tp pointers: rank q's output [batch * seq][N] bf16 (a
 *             mapped peer address for q != rank).  The caller keeps the
 *             mappings valid until the stream has passed this call.
 * Requirements: seq % tp == 0 (else TPL_ERR_INDIVISIBLE), 0 <= rank < tp,
 * 1 <= N <= INT32_MAX, batch * seq <= INT32_MAX (else TPL_ERR_SHAPE); every
 * pointer 2-byte aligned (else TPL_ERR_ALIGN).  16-byte alignment of every
 * buffer and N % 8 == 0 select the vectorised kernel.
 */
tpl_status tpl_reduce_slots_allgather(const void* recv, int32_t tp, int64_t batch, int64_t seq,
                                      int64_t N, const void* bias, const void* residual,
                                      int32_t rank, void* const* peer_y, void* stream);

/*
 * Global argmax of a vocab split over tp GPUs (Tenstorrent LMHead1D: every
 * device's candidates combined at the end).  Rank s ran tpl_lmhead_argmax on
 * its vocab slice (ids local to the slice); after an all-gather of those
 * outputs:
 *   shard_max  device fp32 [tp][B];  shard_idx  device int32 [tp][B], local
 *              ids, -1 for none.  Rank s's global id = s * id_stride + local
 *              (id_stride = the slice size, ceil(V / tp)).
 *   ids        device int32 [B]: the largest logit, ties to the lowest global
 *              id; -1 if no rank has a candidate.
 * Requirements: tp * id_stride <= INT32_MAX.
 */
tpl_status tpl_argmax_merge(const float* shard_max, const int32_t* shard_idx, int32_t tp,
                            int64_t B, int64_t id_stride, int32_t* ids, void* stream);

/*
 * The whole TP MLP block in fp32 in one launch, for latency (nanotron "MLP
 * Module": c_fc column-parallel, activation, c_proj row-parallel with the
 * partial-sum reduction; google-research residual section):
 *   y = act(x W1^T + b1) W2^T (+ b2) (+ residual)
 * computed as the TP shards are.  I is cut into 16 slices, each inside one
 * rank's shard; a cluster of 16 CTAs takes one 8-row token tile and CTA s
 * computes slice s of h (kept in shared memory: h never reaches global
 * memory) and its partial product with W2.  The 16 partials are summed in
 * slice order, which is rank order, then b2 and the residual are added.
 *   x         device fp32 [M][H].
 *   w1        device fp32 [I][H], nn.Linear layout (rank r's shard: rows
 *             r*I/tp .. (r+1)*I/tp - 1).
 *   b1        device fp32 [I] or NULL.
 *   w2        device fp32; rank r's block [H][I/tp] starts at element
 *             H * r * I/tp (the layout tpl_row_linear_reduce takes).
 *   b2        device fp32 [H] or NULL.   residual  device fp32 [M][H] or
 *             NULL; may alias y.
 *   y         device fp32 [M][H].
 * M == 0 is a no-op.  Errors: TPL_ERR_DTYPE (act), TPL_ERR_SHAPE (sizes out
 * of range, more than 65535 tiles of 8 rows), TPL_ERR_INDIVISIBLE
 * (I % tp != 0), TPL_ERR_NULL, TPL_ERR_ALIGN (x, w1, w2, y not 16-byte
 * aligned).  TPL_ERR_UNSUPPORTED for the shapes this kernel does not take:
 * 16 % tp != 0, I % 64 != 0, H % 16 != 0, shared memory
 * 4 * (8 H + (I/16)(H + 4) + H (I/16 + 4) + 8 (I/16 + 4)) bytes above 227 KB
 * (the tiny MLP, H 256 and I 1024, needs 147 KB), or a device that cannot
 * hold a 16-CTA cluster of that size; the caller then runs
 * tpl_column_linear and tpl_row_linear_reduce.
 */
tpl_status tpl_tp_mlp_fp32(const float* x, int64_t M, int64_t H, const float* w1,
                          const float* b1, int64_t I, int32_t tp, tpl_act act, const float* w2,
                          const float* b2, const float* residual, float* y, void* stream);

/*
 * Self-test of the failure path.  (No counterpart on the pages: a diagnostic
 * of this library.)  Launches one thread that waits, with the bounded wait the
 * pipelines use, on an mbarrier nothing arrives on; after limit_ns (1 ns .. 1 s)
 * it records TPL_ERR_TIMEOUT in the status word and returns, leaving the
 * context usable.  waited_us (device int32, or NULL) receives the time waited.
 * tpl_get_device_status then reports and clears TPL_ERR_TIMEOUT.
 */
tpl_status tpl_selftest_wait_timeout(uint64_t limit_ns, int32_t* waited_us, void* stream);

/*
 * Synchronises `stream`, then returns TPL_ERR_TIMEOUT if any kernel of this
 * library on the current device recorded a pipeline timeout since the last
 * call (and clears it), TPL_ERR_CUDA if the stream reports an error, else
 * TPL_OK.
 */
tpl_status tpl_get_device_status(void* stream);

/* Static, human-readable name of a status code. */
const char* tpl_status_string(tpl_status s);

/* Number of tensor-core/CUDA kernels this library enqueued in the calling
 * process since load (host-side count, for launch accounting). */
uint64_t tpl_launch_count(void);

/*
 * Timing records of the tensor-core kernels.  (No counterpart on the pages: a
 * measurement aid of this library.)
 *
 * With a trace buffer installed on the current device, every CTA of the GEMM
 * kernels (tpl_column_linear, tpl_row_linear_reduce and the other GEMM entry
 * points) and of the LM-head kernel appends one tpl_trace_record when it
 * finishes.  t0_ns is %globaltimer when the CTA passed its wait on the kernel
 * before it, t1_ns when it finished, cycles the SM clock cycles (%clock64)
 * between the two; cycles / (t1_ns - t0_ns) is the SM clock the CTA ran at.
 * seq is the launch's number, the value tpl_launch_count returned just before
 * the launch, so the records of one launch share it.
 *
 * buffer     device memory of TPL_TRACE_HEADER_BYTES + capacity * 32 bytes,
 *            16-byte aligned, owned by the caller; NULL removes the buffer
 *            (tracing off, the default).  The call writes the header: a
 *            uint32 record count (starting at 0), then the uint32 capacity.
 *            The count keeps rising past the capacity; the records beyond
 *            it are dropped.
 * capacity   records the buffer holds, 1 .. UINT32_MAX.
 * The call synchronises the device.  Install or remove the buffer while no
 * kernel of this library runs on the device: a running kernel may record
 * into either buffer.  Several threads sharing a device share one buffer.
 * Errors: TPL_ERR_SHAPE (capacity out of range), TPL_ERR_ALIGN (buffer not
 * 16-byte aligned), TPL_ERR_CUDA (the copy or the synchronisation failed).
 */
#define TPL_TRACE_HEADER_BYTES 16
typedef struct tpl_trace_record {
  uint32_t seq;
  uint16_t kind;   /* 1: single-CTA GEMM, 2: CTA-pair GEMM, 3: LM head */
  uint16_t cta;    /* blockIdx.x */
  uint64_t t0_ns;
  uint64_t t1_ns;
  uint64_t cycles;
} tpl_trace_record;
tpl_status tpl_trace_set(void* buffer, int64_t capacity);

#ifdef __cplusplus
}
#endif

#endif /* TPL_H */
