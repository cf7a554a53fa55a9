/*
 * tp_block.h — C ABI of the tensor-parallel Llama decoder block for B200 (sm_100a).
 *
 * One decoder block's decode step, partitioned tensor-parallel into n weight
 * slices that all run as partitions of the same launches on one GPU, plus the
 * 1D / 2D partitioned feed-forward layer and the full multi-layer decode step.
 * Rows may map to cache sequences (prefill chunks, mixed steps), and a block's
 * slices may be spread over processes, one GPU each, with the caller moving the
 * sync buffers between them.
 *
 * Sources for what is computed (pages on the subject, by title and part):
 *   - distributed-llama issue #29, "[Feature Suggest] Tensor Parallellism for
 *     Accelerating LLM": the buildLlama2Arch task list (per-layer order
 *     RmsAttNorm, QuantizeRmsAtt, SyncRmsAtt, Qkv, MultiheadAtt, AttOutput,
 *     QuantizeAtt, SyncAtt, DequantizeAtt, MergeAtt, RmfFfn(Norm), QuantizeRmfFfn,
 *     SyncRmfFfn, Ffn, Ffn2, QuantizeFfn2, SyncFfn2, DequantizeFfn2, MergeFfn2,
 *     NextBlock; then RmsFinal(Norm), Logits, MergeLogits).
 *   - aiterms.tw "Tensor Parallelism" glossary: column split, row split, 2D split
 *     ("core concept") and the FFN procedure with one all-reduce ("how it works").
 *   - CS349E lecture 4 "03_pope_partitioning.py" (Pope et al.), demo1_1d_vs_2d:
 *     1D (split F) versus 2D weight-stationary (split E and F) FFN partitions.
 *
 * Conventions (all entry points):
 *   - Every pointer argument named as a tensor is a DEVICE pointer unless stated.
 *     The caller owns all memory (weights, caches, activations, workspace). The
 *     library never allocates device memory and never synchronises the device;
 *     work is enqueued on `stream` (NULL = the legacy default stream).
 *   - Weights are bf16, stored [out, in] row-major (a PyTorch Linear). A column
 *     split is a contiguous row range of that storage, a row split a contiguous
 *     column range; slices are addressed in place, no re-packing is required.
 *   - Activations and the residual are float32 row-major [B, features].
 *   - KV caches are bf16 [max_batch, n_kv_heads, max_seq, head_dim].
 *   - Slice s of n owns query heads [s*H/n, (s+1)*H/n) and kv heads
 *     [s*Hkv/n, (s+1)*Hkv/n); query head h reads kv head h / (H/Hkv).
 *   - Pointers must be 16-byte aligned. Return value: TP_OK or a tp_status code;
 *     nothing is enqueued when an argument check fails. Faults of kernels already
 *     enqueued surface as CUDA errors at the caller's next synchronisation.
 */
#ifndef TP_BLOCK_H_
#define TP_BLOCK_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TP_API __attribute__((visibility("default")))
#else
#define TP_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* tp_stream; /* a cudaStream_t */

enum tp_status {
  TP_OK = 0,
  TP_EINVAL = 1,      /* a size or flag is out of range or does not divide */
  TP_EWORKSPACE = 2,  /* workspace pointer NULL or smaller than required */
  TP_EARCH = 3,       /* current device is not compute capability 10.0 (B200) */
  TP_ECUDA = 4,       /* a CUDA runtime call or kernel launch failed */
  TP_ENOTSUP = 5,     /* a combination this library does not implement */
  TP_EALIGN = 6,      /* a pointer is not 16-byte aligned */
  TP_ESCRATCH = 7     /* the workspace would exceed the no-allocation entry point's fixed scratch */
};

enum { TP_PART_1D = 1, TP_PART_2D = 2 };
enum { TP_ACT_RELU = 0, TP_ACT_SWIGLU = 1 };
enum { TP_F32 = 0, TP_BF16 = 1 };
enum { TP_MERGE_FAITHFUL = 0, TP_MERGE_FUSED = 1 };

/* Model dimensions (the distributed-llama TransformerSpec, reduced to what one
 * block needs). Requirements checked at create: dim % 128 == 0, head_dim == 128,
 * n_heads / n_kv_heads (query heads per kv head) in {1, 2, 4} or a multiple of 8
 * up to 64 (multi-query attention), H % n == 0, Hkv % n == 0, ffn_dim % (32*n) == 0,
 * 1 <= max_batch <= 64, 1 <= max_seq. */
typedef struct {
  int32_t dim, n_heads, n_kv_heads, head_dim, ffn_dim, vocab, max_batch, max_seq;
  float norm_eps, rope_theta;
} tp_dims;

/* Borrowed device pointers to one block's parameters (the handle keeps them). */
typedef struct {
  const float* attn_norm; /* [dim] float32 RMSNorm gain before attention      */
  const void* wq;         /* bf16 [H*hd, dim]   column split by q-head ranges */
  const void* wk;         /* bf16 [Hkv*hd, dim] column split by kv-head ranges */
  const void* wv;         /* bf16 [Hkv*hd, dim]                               */
  const void* wo;         /* bf16 [dim, H*hd]   row split: slice s reads columns of its heads */
  const float* ffn_norm;  /* [dim] float32 RMSNorm gain before the FFN        */
  const void* w1;         /* bf16 [F, dim]      column split (rows F_s)       */
  const void* w3;         /* bf16 [F, dim]      column split (rows F_s)       */
  const void* w2;         /* bf16 [dim, F]      row split (columns F_s)       */
} tp_block_weights;

/* The same parameters with int8 weights (Pope et al. demo4: decode is bound by the
 * weight bytes, and int8 weights halve them). Each matrix is given as Q8 codes
 * (int8, the same [out, in] layout and slicing as above) and float32 scales
 * [out, in/32]: blocks of 32 consecutive elements along `in`, d = amax/127,
 * codes = x/d rounded half away from zero (the sync-buffer format; tp_quantize_q8
 * of the float32 weights produces exactly this). All pointers 16-byte aligned. */
typedef struct {
  const float* attn_norm;
  const int8_t* wq; const float* wq_d;
  const int8_t* wk; const float* wk_d;
  const int8_t* wv; const float* wv_d;
  const int8_t* wo; const float* wo_d;
  const float* ffn_norm;
  const int8_t* w1; const float* w1_d;
  const int8_t* w3; const float* w3_d;
  const int8_t* w2; const float* w2_d;
} tp_block_weights_q8;

typedef struct tp_block tp_block;

/* Bytes of device workspace a block needs for dims->max_batch rows: the buffers
 * the distributed-llama task list's Sync* steps move (the normalised input in
 * its sync format, the row-split partials) and the kernels' scratch (q, the
 * attention's context splits, the SwiGLU output, the error word and counters).
 * partition: TP_PART_1D or TP_PART_2D (2D applies to the FFN: a gx x gy grid, gx
 * the largest divisor of n with gx*gx <= n splits dim, gy = n/gx splits ffn_dim;
 * attention stays split by heads). sync_quant: 0 = float32 sync buffers,
 * 1 = int8 blocks of 32 with one float32 scale (d = amax/127, codes = x/d rounded
 * half away from zero, clamped to +-127; an all-zero block has d = 0). */
TP_API int tp_block_workspace_bytes(const tp_dims* dims, int n_slices, int partition, int sync_quant,
                             size_t* out_bytes);

/* Validate and build a block handle (host memory only; no device work).
 * workspace: device buffer of at least tp_block_workspace_bytes, 256-byte
 * aligned, owned by the caller, used exclusively by this handle's forwards.
 * Errors: TP_EINVAL, TP_EALIGN, TP_EWORKSPACE, TP_EARCH, TP_ECUDA. */
TP_API int tp_block_create(const tp_dims* dims, int n_slices, int partition, int sync_quant,
                    const tp_block_weights* w, void* workspace, size_t ws_bytes, tp_block** out);

/* A block handle over int8 weights (tp_block_weights_q8). Every slice product
 * then takes Q8 activations as well (the normalised inputs, the attention output
 * before W_O, the SwiGLU output before W2, each quantised in blocks of 32) and
 * runs as integer dot products per block scaled by d_w * d_x, accumulated in
 * float32. Requires partition TP_PART_1D, sync_quant = 1 and ffn_dim % 64 == 0.
 * tp_block_forward on such a handle runs the weight-streaming kernels at every
 * batch, 2 rows per launch: from 6 rows on (where bf16 handles switch to the
 * tensor cores) the weights are read once per 2 rows. Workspace as for
 * tp_block_create.
 * Errors: TP_EINVAL, TP_EALIGN, TP_EWORKSPACE, TP_EARCH, TP_ENOTSUP. */
TP_API int tp_block_create_q8w(const tp_dims* dims, int n_slices, int partition, int sync_quant,
                               const tp_block_weights_q8* w, void* workspace, size_t ws_bytes,
                               tp_block** out);

/* One decode step of the block for `batch` rows (1 <= batch <= max_batch):
 *   x       float32 [batch, dim], read as the residual input and overwritten with
 *           the block output x + attn + ffn.
 *   k_cache, v_cache  bf16 [max_batch, Hkv, max_seq, hd]; positions < pos[b] are
 *           read, position pos[b] is written with the new rotated k and v.
 *   pos     device int32 [batch], 0 <= pos[b] < max_seq (not checked on device:
 *           an out-of-range pos is a caller error).
 * Steps, in the distributed-llama root order: RMSNorm (+Q8) -> q/k/v slice
 * products with RoPE and cache write -> attention per head slice (split over
 * the context, then combined) -> W_O row-split partials [n, batch, dim] ->
 * merge x += sum_s deq(partial_s) in slice order -> RMSNorm (+Q8) -> W1/W3 slice
 * products with SwiGLU -> W2 row-split partials -> merge. */
TP_API int tp_block_forward(tp_block* blk, float* x, void* k_cache, void* v_cache, const int32_t* pos,
                     int batch, tp_stream stream);

/* tp_block_forward for rows that need not own a cache sequence each: row b is a
 * token of sequence seq[b] (device int32 [batch], 0 <= seq[b] < n_seq) at
 * position pos[b], and the caches are bf16 [n_seq, Hkv, max_seq, hd]. Rows of one
 * sequence at consecutive positions are a prefill chunk (Pope et al. demo 2: many
 * tokens of a sequence per step, the regime its weight-gathered layout is for);
 * rows of different sequences mix decode and prefill in one step. Every row's k
 * and v are written before any row's attention runs, so row b attends to
 * positions 0..pos[b] of its sequence including the rows of this step below it:
 * a chunk gives what decoding its tokens one at a time gives. Rows sharing a
 * sequence must have distinct positions (not checked on device). More than
 * max_batch rows run as successive passes of max_batch rows, in row order: a row
 * then also sees the k/v of its sequence's rows in earlier passes, so the rows of
 * a sequence that spans passes must come in increasing position order (a prompt
 * of any length in one call; not checked on device).
 * Errors: TP_EINVAL (also for a rank handle), TP_EALIGN, TP_ECUDA, TP_ENOTSUP. */
TP_API int tp_block_forward_seq(tp_block* blk, float* x, void* k_cache, void* v_cache,
                                const int32_t* pos, const int32_t* seq, int n_seq, int batch,
                                tp_stream stream);

/* Offsets (bytes from the workspace base) and sizes of intermediate buffers,
 * for inspection by tests after a forward. which: 0 xnorm int8 codes [B,dim],
 * 1 xnorm scales float32 [B,dim/32], 2 xnorm float32 [B,dim] (the RMSNorm
 * output before the Q8 round trip; codes and scales are its Q8 form), 3 q
 * (rotated) float32 [B,H*hd], 4 attention output float32 [B,H*hd], 5 partials
 * float32 [n,B,dim], 6 SwiGLU output h float32 [B,F], 7 the kernels' error word
 * (int32 at offset 0: nonzero when a bounded wait in a kernel gave up). Buffers
 * 0-2 hold the last norm a call ran (the FFN's after a whole step). */
TP_API int tp_block_buffer(const tp_block* blk, int which, size_t* offset, size_t* bytes);

TP_API void tp_block_destroy(tp_block* blk);

/* ---------------------------------------------------------------------------
 * The block spread over processes (one GPU each): the distributed-llama task
 * list's nodes, where every node computes its slices' partials and the SyncAtt /
 * SyncFfn2 transfers carry them (quantised when sync_quant is set) to be
 * dequantised and merged (DequantizeAtt, MergeAtt; DequantizeFfn2, MergeFfn2),
 * and the aiterms.tw glossary's "how it works": input replicated, column-split
 * products local, row-split products summed across devices.
 *
 * Rank r of `world` holds slices [r*n/world, (r+1)*n/world) of an n-slice block
 * (requires n % world == 0 and the whole block's rules for n): its weights are
 * those slices only, packed as for tp_block_create -- wq [H/world*hd, dim], wk and
 * wv [Hkv/world*hd, dim], wo [dim, H/world*hd] (the columns of its heads), w1 and
 * w3 [F/world, dim], w2 [dim, F/world], the norm gains whole -- and its KV caches
 * hold its kv heads only, bf16 [max_batch, Hkv/world, max_seq, hd]. `dims`
 * describes the whole block. The residual x [batch, dim] is replicated: every
 * rank passes the same values and all end with the same bits.
 *
 * A decode step is three calls of tp_block_rank_step with phase 0, 1, 2 and the
 * same arguments, with an exchange before phases 1 and 2: the caller gathers the
 * send buffers of all ranks, in rank order, into every rank's receive buffer (an
 * all-gather of tp_block_rank_sync_bytes per rank; rank r's bytes at offset r
 * times that). Phase 0 runs RMSNorm (+Q8), the q/k/v products with RoPE and the
 * cache write, attention and the W_O partials of this rank's slices, and packs
 * them into the send buffer; phase 1 merges the received buffer into x (every
 * slice's partial dequantised and summed in slice order, then added), then runs
 * RMSNorm (+Q8), W1/W3 with SwiGLU and the W2 partials, and packs them; phase 2
 * merges again. Each slice's sync format is float32 [batch, dim], or with
 * sync_quant the int8 codes [batch, dim] followed by the float32 scales
 * [batch, dim/32]. Because every rank merges all n partials in slice order, the
 * result equals the single-process block's merge of the same partials. Phases
 * out of order, or a batch that changes within a step, return TP_EINVAL with
 * nothing enqueued. 1D partition; batch 1..max_batch (<= 5 on the weight-streaming
 * kernels, >= 6 on the tensor-core path, as for tp_block_forward). */
enum { TP_RANK_ATT = 0, TP_RANK_FFN = 1, TP_RANK_OUT = 2 };
#define TP_BUF_SEND 18 /* tp_block_buffer id: this rank's send buffer */
#define TP_BUF_RECV 19 /* tp_block_buffer id: the gathered receive buffer (world x send) */

/* Workspace bytes of rank `rank` of `world` (as tp_block_workspace_bytes, plus
 * the send and receive buffers for max_batch rows). Errors: TP_EINVAL. */
TP_API int tp_block_rank_workspace_bytes(const tp_dims* dims, int n_slices, int sync_quant,
                                         int rank, int world, size_t* out_bytes);

/* A handle for rank `rank` of `world` (weights: this rank's slices, see above).
 * Errors: TP_EINVAL, TP_EALIGN, TP_EWORKSPACE, TP_EARCH, TP_ECUDA. */
TP_API int tp_block_create_rank(const tp_dims* dims, int n_slices, int sync_quant, int rank,
                                int world, const tp_block_weights* w, void* workspace,
                                size_t ws_bytes, tp_block** out);

/* Bytes each rank contributes to an exchange for `batch` rows:
 * (n/world slices) x the slice format's size. Errors: TP_EINVAL (not a rank
 * handle, batch out of range). */
TP_API int tp_block_rank_sync_bytes(const tp_block* blk, int batch, size_t* send_bytes);

/* One phase of a rank's decode step (see above); x, caches and pos as for
 * tp_block_forward, with this rank's kv heads in the caches. Errors: TP_EINVAL,
 * TP_EALIGN, TP_ECUDA. tp_block_forward on a rank handle returns TP_EINVAL. */
TP_API int tp_block_rank_step(tp_block* blk, int phase, float* x, void* k_cache, void* v_cache,
                              const int32_t* pos, int batch, tp_stream stream);

/* Per-stage timing hook. events: host array of n cudaEvent_t handles created by
 * the caller (timing enabled), or NULL to switch the hook off. While set, each
 * tp_block_forward records events[i] on `stream` just before stage i and
 * events[TP_BLOCK_STAGES] after the last stage (n must be TP_BLOCK_STAGES + 1).
 * Stages: 0 RMSNorm(+Q8) + q/k/v products + RoPE + cache write, 1 attention
 * (chunks + combine), 2 W_O partials, 3 merge, 4 RMSNorm(+Q8) + W1/W3 + SwiGLU
 * (2D: stage-1 partials + their merge), 5 W2 partials, 6 final merge. The handle
 * borrows the array; recording works inside stream capture. */
#define TP_BLOCK_STAGES 7
TP_API int tp_block_set_events(tp_block* blk, void* const* events, int n);

/* Persistent block kernel (batch 1-2, 1D partition, GQA group <= 8, n <= 8
 * slices, shapes whose shared-memory plan fits): the whole block forward as one
 * cooperative launch of one CTA per SM, the steps separated by grid barriers,
 * with the weights of the next step streaming into shared memory while the
 * current one finishes. Same arguments and results as the kernel-per-step path.
 * enable: 1 use it for this handle's forwards where the shapes allow, 0 never.
 * The default is 0 unless the environment variable TP_PERSISTENT=1 is set when
 * the handle is created. Errors: TP_EINVAL. */
TP_API int tp_block_set_persistent(tp_block* blk, int enable);

/* Phase trace of the persistent block kernel (batch 1-2, 1D partition), which
 * runs the whole block as one launch and so cannot be split by events. trace:
 * device buffer owned by the caller, at least (SM count) x TP_BLOCK_TRACE_SLOTS
 * x 8 bytes, or NULL to switch tracing off. Each forward that runs the persistent
 * kernel writes, per CTA c, uint64 %globaltimer values (ns) at
 * trace[c * TP_BLOCK_TRACE_SLOTS + k]: k = 0 kernel start; 2p+1 end of phase p
 * and 2p+2 end of the grid barrier after it, for the phases p = 0 q/k/v, 1
 * attention, 2 W_O, 3 W1/W3, 4 W2; 11 end of the final merge; 12 the CTA's last
 * weight or cache copy issued; 13 end of the grid barrier after the merge of the
 * W_O partials (which precedes W1/W3), 14 end of the W1/W3 activation staging
 * (RMSNorm); 15 a duration, not a time: the nanoseconds the CTA's first consumer
 * thread spent waiting for weight stages during W1/W3. While events are set (tp_block_set_events) the
 * block runs as separate kernels and the trace is not written. A forward on the
 * kernel-per-step weight-streaming path (batch <= 5, persistent kernel off)
 * writes instead, for each of its four slice GEMVs g (0 q/k/v, 1 W_O, 2 W1/W3,
 * 3 W2) and CTA c of that launch, trace[c * TP_BLOCK_TRACE_SLOTS + 7g + k]: k = 0
 * start, 1 the previous kernel complete (its wait returned), 2 the RMSNorm scale
 * known, 3 activations staged, 4 the first weight stage arrived, 5 the last stage
 * consumed, 6 end (after the epilogue); for batch > 2 the last launch of each
 * wins; and for its two merges m (0 after W_O, 1 after W2) and merge CTA c < SM
 * count, trace[c * TP_BLOCK_TRACE_SLOTS + 28 + 3m + k]: k = 0 start, 1 the previous
 * kernel complete, 2 end. The persistent kernel uses slots 0-15.
 * Errors: TP_EINVAL (NULL handle, buffer too small). */
#define TP_BLOCK_TRACE_SLOTS 40
TP_API int tp_block_set_trace(tp_block* blk, void* trace, size_t bytes);

/* One block decode step that allocates nothing (no counterpart in the paper: this
 * entry point exists for callers, not for the method).
 *
 * Some callers cannot hand this library a workspace: a plugin running inside a
 * host runtime that owns every byte of device memory through its own pool, or a
 * serving loop that must not call cudaMalloc once it is running (an allocation
 * there would stall the device or is forbidden by the host's allocator). This
 * entry point runs the same kernels as tp_block_create + tp_block_forward, with
 * the same arguments and results, but takes its workspace from one fixed array
 * of TP_NOALLOC_SCRATCH_BYTES (16 MiB) compiled into the library. Every GPU that
 * loads the library holds that array until the process exits. Inputs and outputs
 * are still the caller's: weights, x, the caches and pos as for tp_block_forward.
 *
 * - The first call on a device (with that device current) looks up the array's
 *   device address with cudaGetSymbolAddress; make that first call outside any
 *   stream capture. Every later call made outside stream capture looks it up
 *   again (a device reset moves the array); a call under capture uses the
 *   address of the last call outside it. The call never allocates memory and
 *   frees none.
 * - Configurations whose tp_block_workspace_bytes exceeds the array are refused
 *   with TP_ESCRATCH before anything is enqueued (the 7B block at batch 1 needs
 *   well under 1 MiB; batch 32 of the 70B shape does not fit).
 * - All calls share the one array, which keeps the previous call's contents; the
 *   call zeroes the one word that must start at zero (the kernels' error flag)
 *   on `stream` before its kernels. Calls whose work overlaps on the GPU (other
 *   streams, other host threads) race on the array: serialise them. */
#define TP_NOALLOC_SCRATCH_BYTES (16u << 20)
TP_API int tp_block_forward_noalloc(const tp_dims* dims, int n_slices, int partition,
                                    int sync_quant, const tp_block_weights* w, float* x,
                                    void* k_cache, void* v_cache, const int32_t* pos, int batch,
                                    tp_stream stream);

/* The kernels' error word of the last tp_block_forward_noalloc on the current
 * device (the array is private to the library, so the caller cannot read it
 * from a workspace): copies it into *err (host memory) on `stream`; the value is
 * there once the stream has reached this point. Nonzero means a bounded wait in
 * a kernel gave up and that call's x and cache rows are not valid. Allocates
 * nothing. Errors: TP_EINVAL (err NULL), TP_EARCH, TP_ECUDA. */
TP_API int tp_block_noalloc_error(int* err, tp_stream stream);

/* ------------------------------------------------------------------------- */
/* Partitioned feed-forward layer  Y = act(X W1^T [, X W3^T]) W2^T.            */
/* ------------------------------------------------------------------------- */
typedef struct {
  int32_t batch;      /* tokens B */
  int32_t E, F;       /* model dim and FFN dim */
  int32_t dtype;      /* TP_F32 (X, W float32) or TP_BF16 (X, W bf16) */
  int32_t act;        /* TP_ACT_RELU (two matrices) or TP_ACT_SWIGLU (W1, W3, W2) */
  int32_t partition;  /* TP_PART_1D (n = n_slices over F) or TP_PART_2D (grid_x over E, grid_y over F) */
  int32_t n_slices, grid_x, grid_y;
  int32_t sync_quant; /* 1 = Q8 round trip of every partial before its merge */
  int32_t merge;      /* TP_MERGE_FAITHFUL: every slice's partial formed on its own in
                         float32 (through Q8 with sync_quant) and the partials summed in
                         slice order; TP_MERGE_FUSED: the slices' contraction ranges
                         accumulated in slice order inside the contraction, rounded once
                         (bf16 only, sync_quant must be 0) */
} tp_ffn_desc;

/* Workspace bytes for tp_ffn_forward with this descriptor: the error word, the
 * hidden activations H [B,F] and, where partials are materialised, their float32
 * planes: TP_F32 with TP_MERGE_FAITHFUL (every stage), and the 2D SwiGLU first
 * stage in bf16 (per E-slice). bf16 faithful forms otherwise sum the partials in
 * the tensor-core GEMM's epilogue and need no planes. Errors: TP_EINVAL (sizes
 * that do not divide, see tp_ffn_forward), TP_ENOTSUP. */
TP_API int tp_ffn_workspace_bytes(const tp_ffn_desc* d, size_t* out_bytes);

/* The tensor-parallel FFN Y = act(X W1^T [, X W3^T]) W2^T.
 * Defined by the aiterms.tw "Tensor Parallelism" glossary, "how it works" (the
 * input replicated, Linear1 split by columns, the activation applied locally,
 * Linear2 split by rows, one all-reduce of the partials) and by the Pope et al.
 * lecture script, demo1_1d_vs_2d (1D splits F over n slices; 2D weight-stationary
 * splits E over grid_x and F over grid_y); the ggmlR ggml_pp_dp_forward example
 * fixes the activation after the first stage only.
 * X [B,E], W1 [F,E], W3 [F,E] (NULL unless SwiGLU), W2 [E,F] in d->dtype, all
 * device pointers, row-major, borrowed for the call; Y float32 [B,E] (device)
 * written. 1D: H_s = act(X W1_s^T) per F-slice (column split), P_s = H_s W2_s^T
 * (row split), Y = sum_s P_s in slice order. 2D: stage 1 sums over the E-slices
 * before the activation, stage 2 over the F-slices. With sync_quant every
 * materialised partial passes through the Q8 format before its sum.
 * Requirements: E % (32*grid_x) == 0 and F % (32*n) == 0 (1D) or
 * F % (32*grid_y) == 0 (2D); B >= 1. Errors: TP_EINVAL (sizes, flags, NULL),
 * TP_EALIGN, TP_EWORKSPACE, TP_ENOTSUP (TP_MERGE_FUSED with float32 or with
 * sync_quant), TP_EARCH, TP_ECUDA; nothing is enqueued on an error. */
TP_API int tp_ffn_forward(const tp_ffn_desc* d, const void* X, const void* W1, const void* W3,
                   const void* W2, float* Y, void* workspace, size_t ws_bytes, tp_stream stream);

/* ------------------------------------------------------------------------- */
/* Full decode step: embedding gather, n_layers blocks, final RMSNorm, logits. */
/* ------------------------------------------------------------------------- */
typedef struct tp_model tp_model;

/* Workspace bytes of a model (the distributed-llama layer loop, NextBlock, then
 * RmsFinal, Logits, MergeLogits): one block workspace shared by every layer, the
 * residual and the final normalised rows. Errors: TP_EINVAL. */
TP_API int tp_model_workspace_bytes(const tp_dims* dims, int n_layers, int n_slices, int partition,
                             int sync_quant, size_t* out_bytes);

/* layers: host array of n_layers tp_block_weights (device pointers inside).
 * embed bf16 [vocab, dim]; final_norm float32 [dim]; wcls bf16 [vocab, dim]
 * (the logits are column-split by vocab ranges: each slice writes its own
 * range of the output, so the merge is a concatenation). */
TP_API int tp_model_create(const tp_dims* dims, int n_layers, int n_slices, int partition, int sync_quant,
                    const tp_block_weights* layers, const void* embed, const float* final_norm,
                    const void* wcls, void* workspace, size_t ws_bytes, tp_model** out);

/* tokens device int32 [batch] in [0, vocab); caches bf16
 * [n_layers, max_batch, Hkv, max_seq, hd]; logits float32 [batch, vocab] written. */
/* tp_model_forward with rows mapped to cache sequences (see tp_block_forward_seq):
 * caches bf16 [n_layers, n_seq, Hkv, max_seq, hd]; logits of every row written.
 * More than max_batch rows: successive passes of max_batch rows through every
 * layer, in row order (as tp_block_forward_seq); TP_EALIGN unless max_batch *
 * vocab is a multiple of 4 (each pass's logits rows start 16-byte aligned). */
TP_API int tp_model_forward_seq(tp_model* m, const int32_t* tokens, void* k_cache, void* v_cache,
                                const int32_t* pos, const int32_t* seq, int n_seq, int batch,
                                float* logits, tp_stream stream);

TP_API int tp_model_forward(tp_model* m, const int32_t* tokens, void* k_cache, void* v_cache,
                     const int32_t* pos, int batch, float* logits, tp_stream stream);

/* tp_block_set_persistent for every layer of the model. Errors: TP_EINVAL. */
TP_API int tp_model_set_persistent(tp_model* m, int enable);

TP_API void tp_model_destroy(tp_model* m);

/* ------------------------------------------------------------------------- */
/* Standalone Q8 codec of the sync buffers (same arithmetic as inside the block). */
/* ------------------------------------------------------------------------- */
/* The distributed-llama task list's Quantize* steps (QuantizeRmsAtt, QuantizeAtt,
 * QuantizeRmfFfn, QuantizeFfn2) as one call: x float32 [n] -> q int8 [n],
 * d float32 [n/32], device pointers. Per block of 32 consecutive values:
 * d = amax / 127 (float32, rounded to nearest), q = x / d rounded half away from
 * zero, clamped to +-127; an all-zero block gives d = 0 and zero codes.
 * n % 32 == 0, n >= 0. Errors: TP_EINVAL, TP_EALIGN, TP_EARCH, TP_ECUDA. */
TP_API int tp_quantize_q8(const float* x, int8_t* q, float* d, int64_t n, tp_stream stream);
/* The Dequantize* steps (DequantizeAtt, DequantizeFfn2): q int8 [n],
 * d float32 [n/32] -> x float32 [n], x_i = q_i * d_block (one float32 product).
 * Errors as tp_quantize_q8. */
TP_API int tp_dequantize_q8(const int8_t* q, const float* d, float* x, int64_t n, tp_stream stream);

/* Human-readable name of a status code (static storage). */
TP_API const char* tp_status_string(int status);

/* Library build identifier (static storage), e.g. "tp_block sm_100a". */
TP_API const char* tp_version(void);

#ifdef __cplusplus
}
#endif

#endif /* TP_BLOCK_H_ */
