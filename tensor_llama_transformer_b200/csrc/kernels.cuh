// Kernel argument structs and launchers shared by the host API files.
#pragma once

#include "common.cuh"

namespace tp {

// ------------------------------------------------------------------ merge / codec
// x[b] += sum_{s<n} sync(part_s[b]) in slice order, part_s = the sum of planes
// s*parts .. s*parts+parts-1 of part [n*parts, B, dim] (a slice's contraction
// split further by the GEMM). With ssq != nullptr the sum of squares of every
// 128-value chunk of the new row is written too: ssq[b][chunk] (merge_ssq_parts(dim)
// of them; each warp's squares summed by warp_sum and the chunk's four warp sums in
// order, in both merge kernels, so that both give the next RMSNorm the same bits).
// dim % 128 == 0, parts <= 2.
// Optional %globaltimer stamps of merge CTA c < rows: stamps[c * stride + k], k = 0
// start, 1 the previous kernel complete, 2 end.
struct MergeTrace {
  unsigned long long* stamps;
  int stride, rows;
};
// late: the next kernel may launch only once every CTA's partials have been loaded
// (its weight stream then does not compete with those loads); else at the start.
int launch_merge(float* x, const float* part, int n, int B, int dim, int quant, float* ssq,
                 cudaStream_t s, int parts = 1, MergeTrace trace = MergeTrace{}, int late = 0);
inline int merge_ssq_parts(int dim) { return dim / 128; }
// One slice's partial in the sync format for B rows: float32 [B, dim], or with Q8
// the codes int8 [B, dim] followed by the scales float32 [B, dim/32].
__host__ __device__ inline int64_t sync_slice_bytes(int B, int dim, int quant) {
  return quant ? (int64_t)B * dim + (int64_t)B * (dim / 32) * 4 : (int64_t)B * dim * 4;
}
// Rank side of a block spread over processes: pack the n_local slices' partials
// (planes as for launch_merge) into their sync format, slice after slice; and
// merge a gathered buffer of n slices in that format into x (slice order, ssq as
// launch_merge). dim % 128 == 0.
int launch_sync_pack(const float* part, int n_local, int parts, int B, int dim, int quant,
                     uint8_t* out, cudaStream_t s);
int launch_merge_sync(float* x, const uint8_t* sync, int n, int B, int dim, int quant, float* ssq,
                      cudaStream_t s);
int launch_quantize(const float* x, int8_t* q, float* d, int64_t n, cudaStream_t s);
int launch_dequantize(const int8_t* q, const float* d, float* x, int64_t n, cudaStream_t s);

// ------------------------------------------------------------------ slice GEMV
enum GemvEpi { EPI_PLAIN = 0, EPI_SWIGLU = 1, EPI_QKV = 2 };

struct GemvArgs {
  // weights: up to three bf16 matrices [rows_i, ldw] stacked in row space (QKV),
  // or two matrices read row for row together (SwiGLU: W1 row f with W3 row f).
  const uint16_t* w[3];
  int rows[3];
  int64_t ldw;   // row stride in elements (= full input width K)
  // int8 weights: w[i] then holds Q8 codes (int8, same layout) and wd[i] their
  // float32 scales [rows_i, ldw / 32]; the activations enter as Q8 codes too and
  // the products are integer dot products per 32-value block, scaled by d_w d_x.
  const float* wd[3];
  // input taken from the attention's context splits instead of x (W_O on the
  // weight-streaming path): partial outputs [B, H, att_nsplit, hd] and (m, l)
  // [B, H, att_nsplit, 2], combined while staging; the CTA that owns a segment's
  // first row writes the combined row to att_out [B, H*hd].
  const float* att_po;
  const float* att_pml;
  int att_nsplit;
  float* att_out;
  int Ks;        // contraction length of one segment
  int nseg;      // number of segments: segment s reads columns [s*Ks, (s+1)*Ks)
  // input: float32 x [B, ldx] or Q8 (xq [B, ldx], xd [B, ldx/32]); with `gain`
  // set, x is a residual and the input is RMSNorm(x) * gain (+Q8 when quant),
  // computed in the prologue; the first CTA of each segment then writes the
  // shared buffer (xq_out/xd_out: the Q8 codes and scales; xn_out: the float32
  // RMSNorm output before any Q8 round trip; each nullable).
  const float* x;
  const int8_t* xq;
  const float* xd;
  int ldx;
  const float* gain;
  float eps;
  int quant;
  const float* ssq;  // optional per-row partial sums of squares of x [B][ssq_parts] (fixed order)
  int ssq_parts;
  int8_t* xq_out;
  float* xd_out;
  float* xn_out;
  int b0, nb;    // batch rows [b0, b0+nb) handled by this launch
  // EPI_PLAIN / EPI_SWIGLU output: out[seg*out_seg + b*ldo + row]
  float* out;
  uint16_t* out_bf16;  // optional bf16 copy, same indexing
  int64_t out_seg;
  int ldo;
  // EPI_QKV
  float* qout;   // rotated q [B, H*hd]
  uint16_t* kc;  // caches [sequences, Hkv, max_seq, hd]
  uint16_t* vc;
  const int32_t* pos;
  const int32_t* seq;  // cache sequence of each row (nullable: row b uses sequence b)
  int n_heads, n_kv_heads, max_seq;
  float theta;
  // optional %globaltimer stamps (ns) of CTA c at trace[c * trace_stride + k]:
  // k = 0 start, 1 previous kernel complete, 2 RMSNorm scale known, 3 activations
  // staged, 4 first ring stage arrived, 5 last ring stage consumed, 6 end
  unsigned long long* trace;
  int trace_stride;
  int* err;  // device error flag, set when a bounded wait gives up (nullable)
};


// Shared-memory plan of the GEMV (host computes, kernel reads): NC consumer
// warps, row pairs per stage (each pair split over `split` warps), ring depth,
// and the offsets of the ring, the staged activations, the per-row partial
// results and the mbarriers.
struct GemvPlan {
  int nc;
  int pairs;
  int split;
  int pw;  // row pairs per warp and stage (2 with 16 pairs per stage)
  int nstage;
  int cta_rows;
  // row-split bf16 weights read through a 3D tensor map (the kernel's wmap): boxes of
  // map_box consecutive rows of one segment (map_nchunk chunks of the map's inner
  // width), one TMA per box instead of one bulk copy per row; 0: bulk copies
  int map_box, map_nchunk;
  size_t ring_off, x_off, res_off, bar_off, total;
};

int launch_gemv(const GemvArgs& a, int epi, cudaStream_t s);

// ------------------------------------------------------------------ attention
struct AttnArgs {
  const float* q;       // rotated q [B, H*hd]
  const uint16_t* kc;   // [nseq, Hkv, max_seq, hd] bf16
  const uint16_t* vc;
  const int32_t* pos;   // [B]
  const int32_t* seq;   // [B] cache sequence of each row (nullable: row b)
  int nseq;             // sequences in the caches (with seq; else B)
  int B, H, Hkv, max_seq;
  int nchunk;           // capacity of the partial buffers in context splits
  float* part_o;        // [B, H, nsplit, hd] unnormalised partial outputs (nsplit <= nchunk)
  float* part_ml;       // [B, H, nsplit, 2] running max and sum
  float* att;           // [B, H*hd] combined output
  uint16_t* att_bf16;   // optional hi/lo bf16 pairs [2B, H*hd] (rows 2b, 2b+1)
  int nsplit;           // context splits (0: attention_nsplit's choice)
  int* err;             // device error flag (bounded waits)
};

// combine = false leaves the splits' partials for the consumer to combine (the
// W_O GEMV's staging on the weight-streaming path).
int launch_attention(const AttnArgs& a, cudaStream_t s, bool combine = true);
// Context splits per (batch row, kv head) the attention uses for these shapes.
int attention_nsplit(int B, int H, int Hkv, int max_seq);
// Largest number of context splits any launch over max_seq positions uses.
int attention_max_splits(int max_seq);

// ------------------------------------------------------------------ batched decode
// Batches at least this large run the slice products on the tcgen05 GEMM (the
// weights as the M operand, the batch as N); smaller ones on the ring GEMV.
constexpr int kTcMinBatch = 6;

struct NormRowsArgs {
  const float* x;      // residual [B, dim]
  const float* gain;   // [dim]
  const float* ssq;    // optional per-row partial sums of squares [B][ssq_parts]
  int ssq_parts;
  int dim;
  float eps;
  int quant;
  int8_t* xq;          // Q8 codes [B, dim] (nullable)
  float* xd;           // Q8 scales [B, dim/32] (nullable)
  float* xn;           // float32 RMSNorm output, before any Q8 round trip (nullable)
  uint16_t* xb;        // the value the slices read (after Q8 when quant) as hi/lo bf16
                       // pairs [2B, dim] (tensor-core operand)
};
int launch_norm_rows(const NormRowsArgs& a, int batch, cudaStream_t s);

struct QkvFinalizeArgs {
  const float* plane;  // [parts][batch][qd + 2 kd]
  int parts, batch, qd, kd;
  const int32_t* pos;
  const int32_t* seq;  // cache sequence of each row (nullable: row b)
  float theta;
  float* q;            // [batch, qd]
  uint16_t* kc;
  uint16_t* vc;
  int n_kv_heads, max_seq;
};
int launch_qkv_finalize(const QkvFinalizeArgs& a, cudaStream_t s);
// h = silu(a) * g from planes [parts][batch][2F] (a = columns [0, F), g = [F, 2F),
// each the sum of the parts in order), with its hi/lo bf16 pair rows.
int launch_swiglu_finalize(const float* plane, int parts, int F, int batch, float* h,
                           uint16_t* hb, cudaStream_t s);

// ------------------------------------------------------------------ persistent block
// One weight-streaming phase of the persistent block kernel: the rows of up to
// three matrices (q/k/v stacked; W1/W3 interleaved row for row), contracted over
// nseg segments of Ks columns. pairs/split are filled by the plan.
struct BpGemv {
  const uint16_t* w[3];
  int rows[3];
  int64_t ldw;
  int Ks, nseg, rps;  // rps: virtual rows per segment
  int pairs, split;   // row pairs per ring stage; warps per pair
  int pw;             // row pairs per warp and stage (1, or 2 with 16 pairs per stage)
};

struct BpArgs {
  int D, F, H, Hkv, QD, n, quant, max_seq, nb, nchunk;
  float eps, theta;
  const float* attn_norm;
  const float* ffn_norm;
  BpGemv g[4];          // q/k/v, W_O, W1/W3, W2
  float* x;             // residual [nb, D], overwritten with the block output
  uint16_t* kc;         // caches [maxB, Hkv, max_seq, hd]
  uint16_t* vc;
  const int32_t* pos;
  int8_t* xq;           // published sync buffers (Q8 codes, scales, float32 values)
  float* xd;
  float* xn;
  float* q;             // rotated q [nb, QD]
  float* part_o;        // attention splits [nb, H, nchunk, hd] and [nb, H, nchunk, 2]
  float* part_ml;
  float* att;           // attention output [nb, QD]
  float* part;          // row-split partials [n, nb, D] (W_O, then W2)
  float* xmid;          // x + attention branch [nb, D]
  float* ssq;           // sums of squares of x_mid per 128 values [nb][D/128]
  float* h;             // SwiGLU output [nb, F]
  int* err;             // error word
  unsigned* bar;        // grid barrier counters (two words, zero between launches)
  unsigned long long* trace;  // optional [grid][kBpTraceSlots] %globaltimer stamps (ns)
  int grid;
  uint32_t ring_bytes, xs_off, res_off, smem_total;
};
// Trace stamps per CTA: 0 start, then for each phase A..F its end (2k+1) and,
// for A..E, the end of the grid barrier after it (2k+2); 12 the producer's last
// issue; 13 the end of the barrier after the W_O-partial merge, 14 the end of
// the activation staging of phase D; 15 the time (ns) thread 0 waited for ring
// stages during phase D.
constexpr int kBpTraceSlots = 16;
static_assert(kBpTraceSlots <= TP_BLOCK_TRACE_SLOTS, "trace layout");
// Fills the launch plan (grid, shared-memory layout, rows per stage); false when
// the shapes rule the persistent kernel out.
bool plan_block_persistent(BpArgs& a, int nb_max);
// Whether handles use the persistent kernel unless told otherwise (TP_PERSISTENT=1).
bool persistent_default();
int launch_block_persistent(const BpArgs& a, int nb_max, cudaStream_t s);

// One block forward over a caller-provided workspace with a handle on the stack
// (api.cu); zeroes the kernels' error word in the workspace first.
int block_forward_on_workspace(const tp_dims* dims, int n_slices, int partition, int sync_quant,
                               const tp_block_weights* w, void* workspace, size_t ws_bytes,
                               float* x, void* k_cache, void* v_cache, const int32_t* pos,
                               int batch, cudaStream_t stream);

}  // namespace tp
