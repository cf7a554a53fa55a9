// Host side of the C ABI declared in include/tp_block.h: argument checks,
// workspace layout and the launch sequence of a block, a model and an FFN.
#include <cstdlib>
#include <mutex>
#include <new>

#include "ffn.cuh"
#include "gemm_tc.cuh"
#include "kernels.cuh"

namespace tp {

// ------------------------------------------------------------------ device info
namespace {
constexpr int kMaxDev = 64;
int g_arch[kMaxDev];  // 0 unknown, 1 sm_100, 2 other
int g_sms[kMaxDev];
}  // namespace

int device_check() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return TP_ECUDA;
  if (g_arch[dev] == 0) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return TP_ECUDA;
    g_sms[dev] = sms;
    g_arch[dev] = (major == 10 && minor == 0) ? 1 : 2;
  }
  return g_arch[dev] == 1 ? TP_OK : TP_EARCH;
}

int set_smem_once(const void* kernel, int bytes) {
  struct Entry {
    const void* fn;
    int dev;
    int bytes;
  };
  static Entry tab[256];
  static int used = 0;
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return TP_ECUDA;
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < used; ++i)
    if (tab[i].fn == kernel && tab[i].dev == dev && tab[i].bytes >= bytes) return TP_OK;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
      cudaSuccess)
    return TP_ECUDA;
  for (int i = 0; i < used; ++i)
    if (tab[i].fn == kernel && tab[i].dev == dev) {
      tab[i].bytes = bytes;
      return TP_OK;
    }
  if (used < 256) tab[used++] = Entry{kernel, dev, bytes};
  return TP_OK;
}

bool pdl_enabled() {
  static const bool on = [] {
    const char* v = getenv("TP_PDL");
    return !(v && v[0] == '0');
  }();
  return on;
}

int num_sms() {
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= kMaxDev || g_sms[dev] == 0) device_check();
  return (dev >= 0 && dev < kMaxDev && g_sms[dev] > 0) ? g_sms[dev] : 148;
}

namespace {

size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

// ------------------------------------------------------------------ block layout
enum Buf {
  BUF_XQ = 0, BUF_XD, BUF_XN, BUF_Q, BUF_ATT, BUF_PART, BUF_H, BUF_ERR, BUF_PO, BUF_PML,
  BUF_PA, BUF_PB, BUF_SSQ, BUF_XB, BUF_ATTB, BUF_HB, BUF_PLANE, BUF_XMID, BUF_SEND, BUF_RECV,
  BUF_COUNT
};
static_assert(BUF_SEND == TP_BUF_SEND && BUF_RECV == TP_BUF_RECV, "buffer ids of the C ABI");
// BUF_ERR (16 bytes, placed first: byte 0 of every block workspace): the int
// error word at byte 0; the persistent kernel's two grid barrier counters at
// bytes 8 and 12 (zero between launches). The handle's first forward zeroes all.
constexpr size_t kCountersOff = 8;

// Largest contraction splits of the batched-decode GEMMs (the planes are sized for them).
constexpr int kQkvMaxParts = 8, kW13MaxParts = 4, kW2MaxParts = 2;

struct Layout {
  size_t off[BUF_COUNT];
  size_t size[BUF_COUNT];
  size_t total;
};

struct Cfg {
  tp_dims d;  // for a rank block: this rank's share (H, Hkv, ffn_dim divided by world)
  int n, partition, quant, gx, gy, nchunk;
  int rank, world;  // world 0: the whole block; else this process holds n of n * world slices
};

void grid2d(int n, int* gx, int* gy) {
  int best = 1;
  for (int v = 1; v * v <= n; ++v)
    if (n % v == 0) best = v;
  *gx = best;
  *gy = n / best;
}

int check_cfg(const tp_dims* d, int n, int partition, int quant, Cfg* c) {
  if (!d || !c) return TP_EINVAL;
  if (n < 1 || (partition != TP_PART_1D && partition != TP_PART_2D) || (quant != 0 && quant != 1))
    return TP_EINVAL;
  if (d->dim <= 0 || d->dim % 128 != 0) return TP_EINVAL;
  if (d->head_dim != kHeadDim) return TP_ENOTSUP;
  if (d->n_heads <= 0 || d->n_kv_heads <= 0 || d->n_heads % d->n_kv_heads != 0) return TP_EINVAL;
  const int G = d->n_heads / d->n_kv_heads;  // query heads per kv head (GQA / MQA)
  if (G != 1 && G != 2 && G != 4 && !(G % 8 == 0 && G <= 64)) return TP_ENOTSUP;
  if (d->n_heads % n != 0 || d->n_kv_heads % n != 0) return TP_EINVAL;
  if (d->ffn_dim <= 0 || d->ffn_dim % (32 * n) != 0) return TP_EINVAL;
  if (d->max_batch < 1 || d->max_batch > 64 || d->max_seq < 1) return TP_EINVAL;
  if (!(d->norm_eps >= 0.f) || !(d->rope_theta > 0.f)) return TP_EINVAL;
  c->d = *d;
  c->n = n;
  c->partition = partition;
  c->quant = quant;
  if (partition == TP_PART_2D) {
    grid2d(n, &c->gx, &c->gy);
    if (d->dim % (32 * c->gx) != 0 || d->ffn_dim % (32 * c->gy) != 0) return TP_EINVAL;
  } else {
    c->gx = 1;
    c->gy = n;
  }
  c->nchunk = attention_max_splits(d->max_seq);
  c->rank = 0;
  c->world = 0;
  return TP_OK;
}

// A rank's share of an n-slice block spread over `world` processes: slices
// [rank n/world, (rank+1) n/world) with their q/kv heads and ffn rows, i.e. a
// block of n/world slices over H/world heads, Hkv/world kv heads and F/world
// ffn rows; dim and the norms are whole.
int check_rank_cfg(const tp_dims* d, int n, int quant, int rank, int world, Cfg* c) {
  if (!d || world < 1 || rank < 0 || rank >= world || n < 1 || n % world != 0) return TP_EINVAL;
  int rc = check_cfg(d, n, TP_PART_1D, quant, c);  // the whole block's rules
  if (rc) return rc;
  tp_dims local = *d;
  local.n_heads /= world;
  local.n_kv_heads /= world;
  local.ffn_dim /= world;
  rc = check_cfg(&local, n / world, TP_PART_1D, quant, c);
  if (rc) return rc;
  c->rank = rank;
  c->world = world;
  return TP_OK;
}

Layout block_layout(const Cfg& c) {
  const size_t B = c.d.max_batch, D = c.d.dim, F = c.d.ffn_dim;
  const size_t QD = (size_t)c.d.n_heads * c.d.head_dim;
  Layout L{};
  L.size[BUF_XQ] = B * D;
  L.size[BUF_XD] = B * (D / 32) * 4;
  L.size[BUF_XN] = B * D * 4;
  L.size[BUF_Q] = B * QD * 4;
  L.size[BUF_ATT] = B * QD * 4;
  // row-split partials: n slices (x kW2MaxParts contraction parts on the tensor path)
  L.size[BUF_PART] = (size_t)c.n * (c.d.max_batch >= kTcMinBatch ? kW2MaxParts : 1) * B * D * 4;
  L.size[BUF_H] = B * F * 4;
  L.size[BUF_ERR] = 16;
  L.size[BUF_PO] = B * c.d.n_heads * (size_t)c.nchunk * c.d.head_dim * 4;
  L.size[BUF_PML] = B * c.d.n_heads * (size_t)c.nchunk * 2 * 4;
  const size_t pa = c.partition == TP_PART_2D ? (size_t)c.gx * B * F * 4 : 0;
  L.size[BUF_PA] = pa;
  L.size[BUF_PB] = pa;
  // per-row sums of squares: merge pieces of 512 values, or (persistent kernel) 128
  L.size[BUF_SSQ] = B * (size_t)(c.d.dim / 128) * 4;
  L.size[BUF_XMID] = B * D * 4;  // x + attention branch (persistent kernel)
  if (c.world > 0) {  // rank block: its slices' sync buffers out, every rank's in
    const size_t chunk = (size_t)sync_slice_bytes(c.d.max_batch, c.d.dim, c.quant);
    L.size[BUF_SEND] = (size_t)c.n * chunk;
    L.size[BUF_RECV] = (size_t)c.n * c.world * chunk;
  }
  // batched decode (tensor-core path): bf16 operands and the float32 product planes
  if (c.d.max_batch >= kTcMinBatch) {
    const size_t KD = (size_t)c.d.n_kv_heads * c.d.head_dim;
    L.size[BUF_XB] = 2 * B * D * 2;  // hi/lo bf16 pairs
    L.size[BUF_ATTB] = 2 * B * QD * 2;
    L.size[BUF_HB] = 2 * B * F * 2;
    const size_t qkv = kQkvMaxParts * B * (QD + 2 * KD) * 4;  // contraction parts
    const size_t w13 = kW13MaxParts * B * 2 * F * 4;
    L.size[BUF_PLANE] = qkv > w13 ? qkv : w13;
  }
  // the error word first, at byte 0 of the workspace; then the others in id order
  size_t o = align256(L.size[BUF_ERR]);
  L.off[BUF_ERR] = 0;
  for (int i = 0; i < BUF_COUNT; ++i) {
    if (i == BUF_ERR) continue;
    L.off[i] = o;
    o += align256(L.size[i]);
  }
  L.total = o;
  return L;
}

}  // namespace
}  // namespace tp

using namespace tp;

struct tp_block {
  Cfg c;
  Layout L;
  tp_block_weights w;
  uint8_t* ws;
  size_t ws_bytes;
  void* const* events;  // optional per-stage timing events (borrowed)
  bool bar_ready;       // the counters of BUF_ERR (grid barriers, merge pieces) known to be zero
  unsigned long long* trace;  // optional phase trace (persistent kernel, or the four slice GEMVs)
  int persistent;       // use the persistent kernel where the shapes allow (batch 1-2, 1D)
  bool wq8;             // int8 weights: w holds the codes, wd their scales
  const float* wd_q;
  const float* wd_k;
  const float* wd_v;
  const float* wd_o;
  const float* wd_1;
  const float* wd_3;
  const float* wd_2;
  int phase_next;   // rank block: the phase tp_block_rank_step expects next
  int phase_batch;  // rank block: the batch of the step in progress
};

struct tp_model {
  tp_dims d;
  int n_layers;
  tp_block* blocks;  // n_layers handles sharing one block workspace
  const void* embed;
  const float* final_norm;
  const void* wcls;
  float* x;    // residual [max_batch, dim]
  float* xnf;  // final normed rows [max_batch, dim]
};

namespace tp_api {

template <typename T>
T* at(const tp_block* b, int buf) {
  return reinterpret_cast<T*>(b->ws + b->L.off[buf]);
}

// RMSNorm(+Q8) of the residual rows computed in a GEMV's prologue; the first
// CTA of each segment publishes the shared buffer (Q8 codes + scales, or fp32).
void set_norm_input(const tp_block* b, GemvArgs& a, const float* x, const float* gain) {
  a.x = x;
  a.ldx = b->c.d.dim;
  a.gain = gain;
  a.eps = b->c.d.norm_eps;
  a.quant = b->c.quant;
  if (b->c.quant) {
    a.xq_out = at<int8_t>(b, BUF_XQ);
    a.xd_out = at<float>(b, BUF_XD);
  }
  a.xn_out = at<float>(b, BUF_XN);  // the float32 RMSNorm output (before Q8)
}

// Records the caller's timing event before `stage`. Inside stream capture the
// record must be an external event node (a plain record would only become a
// dependency edge of the graph and never be timestamped).
int stage_mark(const tp_block* blk, int stage, cudaStream_t s) {
  if (!blk->events) return TP_OK;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cap) != cudaSuccess) return TP_ECUDA;
  cudaEvent_t ev = static_cast<cudaEvent_t>(blk->events[stage]);
  const cudaError_t e = cap == cudaStreamCaptureStatusActive
                            ? cudaEventRecordWithFlags(ev, s, cudaEventRecordExternal)
                            : cudaEventRecord(ev, s);
  return e == cudaSuccess ? TP_OK : TP_ECUDA;
}

// a6 / a10. Whole block: x += the slice partials (planes of `part`), summed in
// slice order through the sync format. Rank block: the same over the gathered
// sync buffer, which holds every rank's slices in slice order.
// m: 0 the merge after W_O, 1 the merge after W2 (trace slots 28 + 3m .. 30 + 3m).
int merge_step(tp_block* blk, float* x, const float* part, int nseg, int parts, int batch,
               cudaStream_t s, int m) {
  const Cfg& c = blk->c;
  float* ssq = at<float>(blk, BUF_SSQ);
  if (c.world == 0) {
    MergeTrace t{};
    if (blk->trace) {
      t.stamps = blk->trace + 28 + 3 * m;
      t.stride = TP_BLOCK_TRACE_SLOTS;
      t.rows = num_sms();
    }
    // int8 weights: the next GEMV's weight stream starts after the merge's loads (the
    // int8 block measured 66.0 against 66.9 us; the bf16 blocks are faster with the
    // stream overlapping the merge: C2 89.9 against 90.4 us)
    return launch_merge(x, part, nseg, batch, c.d.dim, c.quant, ssq, s, parts, t, blk->wq8 ? 1 : 0);
  }
  return launch_merge_sync(x, at<uint8_t>(blk, BUF_RECV), c.n * c.world, batch, c.d.dim, c.quant,
                           ssq, s);
}

// Trace slots 7g .. 7g+6 of every CTA for the slice GEMV g (0 q/k/v, 1 W_O,
// 2 W1/W3, 3 W2) when a trace buffer is set.
void set_gemv_trace(const tp_block* blk, GemvArgs& a, int g) {
  if (!blk->trace) return;
  a.trace = blk->trace + 7 * g;
  a.trace_stride = TP_BLOCK_TRACE_SLOTS;
}

// End of a rank block's phase 0 / 1: this rank's partials into its send buffer.
int pack_step(tp_block* blk, const float* part, int parts, int batch, cudaStream_t s) {
  const Cfg& c = blk->c;
  return launch_sync_pack(part, c.n, parts, batch, c.d.dim, c.quant, at<uint8_t>(blk, BUF_SEND), s);
}

// Contraction parts for a batched-decode GEMM of `tiles` 128-row output tiles
// (per existing segment) over K: the persistent GEMM gives each SM ceil(tiles *
// parts / SMs) tiles of K / parts, and every extra part adds a float32 plane
// [batch, rows] that is written and read back. Picks the power of two <= pmax
// (with K / parts a multiple of 64) that minimises the busiest SM's weight bytes
// plus its share of the planes' traffic.
int tc_split(int64_t tiles, int64_t K, int64_t rows_total, int batch, int pmax) {
  const int64_t sms = num_sms();
  int best = 1;
  double best_cost = -1.0;
  for (int p = 1; p <= pmax; p *= 2) {
    if (K % (64 * p) != 0 && p > 1) break;
    const double main = (double)((tiles * p + sms - 1) / sms) * 128.0 * (double)(K / p) * 2.0;
    const double planes = 2.0 * p * (double)batch * (double)rows_total * 4.0 / (double)sms;
    const double cost = main + planes;
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = p;
    }
  }
  return best;
}


// The batched form of the block: the same steps, with the slice products on the
// tcgen05 GEMM (weights = M operand, batch = N) writing float32 planes, small
// kernels for the norms and epilogues, and the same attention and merges.
// phase: -1 the whole step; 0 / 1 / 2 a rank block's steps (tp_block_rank_step).
int block_forward_tc(tp_block* blk, float* x, void* kc, void* vc, const int32_t* pos, int batch,
                     cudaStream_t s, bool chained, int phase, const int32_t* seq, int nseq) {
  const Cfg& c = blk->c;
  const tp_dims& d = c.d;
  const int D = d.dim, F = d.ffn_dim, H = d.n_heads, Hkv = d.n_kv_heads, hd = d.head_dim;
  const int QD = H * hd, KD = Hkv * hd;
  int rc;
  float* part = at<float>(blk, BUF_PART);
  float* plane = at<float>(blk, BUF_PLANE);
  uint16_t* xb = at<uint16_t>(blk, BUF_XB);
  int* err = at<int>(blk, BUF_ERR);
  auto norm = [&](const float* gain, const float* ssq) -> int {
    NormRowsArgs n{};
    n.x = x;
    n.gain = gain;
    n.ssq = ssq;
    n.ssq_parts = merge_ssq_parts(D);
    n.dim = D;
    n.eps = d.norm_eps;
    n.quant = c.quant;
    n.xq = c.quant ? at<int8_t>(blk, BUF_XQ) : nullptr;
    n.xd = c.quant ? at<float>(blk, BUF_XD) : nullptr;
    n.xn = at<float>(blk, BUF_XN);
    n.xb = xb;
    return launch_norm_rows(n, batch, s);
  };
  auto gemm = [&](const void* A0, int m0, const void* A1, int m1, const void* A2, int m2, int nA,
                  int64_t lda, const uint16_t* Bop, int K, int nseg, float* out, int64_t rows) {
    TcGemm g{};
    g.A[0] = A0;
    g.A[1] = A1;
    g.A[2] = A2;
    g.Am[0] = m0;
    g.Am[1] = m1;
    g.Am[2] = m2;
    g.nA = nA;
    g.lda = lda;
    g.B = Bop;
    g.ldb = lda;
    g.N = 2 * batch;  // hi/lo row pairs of the activations
    g.K = K;
    g.nseg = nseg;
    g.epi = TC_EPI_STORE_T_PAIRS_F32;
    g.out = out;
    g.ldo = rows;
    g.out_seg = (int64_t)batch * rows;
    g.err = err;
    g.indep = TC_INDEP_A;  // the weights
    return launch_tc_gemm(g, s);
  };

  const int nseg2 = c.partition == TP_PART_1D ? c.n : c.gy;
  int p2 = 1;
  if (phase <= 0) {
    // a1-a4
    if ((rc = stage_mark(blk, 0, s))) return rc;
    if ((rc = norm(blk->w.attn_norm, chained ? at<float>(blk, BUF_SSQ) : nullptr))) return rc;
    const int qkv_tiles = (QD + 127) / 128 + 2 * ((KD + 127) / 128);
    const int parts = tc_split(qkv_tiles, D, QD + 2 * KD, batch, kQkvMaxParts);
    if ((rc = gemm(blk->w.wq, QD, blk->w.wk, KD, blk->w.wv, KD, 3, D, xb, D / parts, parts, plane,
                   QD + 2 * KD)))
      return rc;
    {
      QkvFinalizeArgs f{};
      f.plane = plane;
      f.parts = parts;
      f.batch = batch;
      f.qd = QD;
      f.kd = KD;
      f.pos = pos;
      f.seq = seq;
      f.theta = d.rope_theta;
      f.q = at<float>(blk, BUF_Q);
      f.kc = static_cast<uint16_t*>(kc);
      f.vc = static_cast<uint16_t*>(vc);
      f.n_kv_heads = Hkv;
      f.max_seq = d.max_seq;
      if ((rc = launch_qkv_finalize(f, s))) return rc;
    }
    // a4
    if ((rc = stage_mark(blk, 1, s))) return rc;
    {
      AttnArgs a{};
      a.q = at<float>(blk, BUF_Q);
      a.kc = static_cast<const uint16_t*>(kc);
      a.vc = static_cast<const uint16_t*>(vc);
      a.pos = pos;
      a.seq = seq;
      a.nseq = nseq;
      a.B = batch;
      a.H = H;
      a.Hkv = Hkv;
      a.max_seq = d.max_seq;
      a.nchunk = c.nchunk;
      a.part_o = at<float>(blk, BUF_PO);
      a.part_ml = at<float>(blk, BUF_PML);
      a.att = at<float>(blk, BUF_ATT);
      a.att_bf16 = at<uint16_t>(blk, BUF_ATTB);
      a.err = err;
      if ((rc = launch_attention(a, s))) return rc;
    }
    // a5: W_O row-split partials (segment s = slice s's head columns)
    if ((rc = stage_mark(blk, 2, s))) return rc;
    if ((rc = gemm(blk->w.wo, D, nullptr, 0, nullptr, 0, 1, QD, at<uint16_t>(blk, BUF_ATTB), QD / c.n,
                   c.n, part, D)))
      return rc;
    if (phase == 0) return pack_step(blk, part, 1, batch, s);
  }
  if (phase <= 1) {
    // a6 (a rank block: the merge of the gathered buffer)
    if ((rc = stage_mark(blk, 3, s))) return rc;
    if ((rc = merge_step(blk, x, part, c.n, 1, batch, s, 0))) return rc;
    // a7-a8
    if ((rc = stage_mark(blk, 4, s))) return rc;
    if ((rc = norm(blk->w.ffn_norm, at<float>(blk, BUF_SSQ)))) return rc;
    float* hbuf = at<float>(blk, BUF_H);
    uint16_t* hb = at<uint16_t>(blk, BUF_HB);
    if (c.partition == TP_PART_1D) {
      const int p13 = tc_split(2 * ((F + 127) / 128), D, 2 * F, batch, kW13MaxParts);
      if ((rc = gemm(blk->w.w1, F, blk->w.w3, F, nullptr, 0, 2, D, xb, D / p13, p13, plane, 2 * F)))
        return rc;
      if ((rc = launch_swiglu_finalize(plane, p13, F, batch, hbuf, hb, s))) return rc;
    } else {
      float* pa = at<float>(blk, BUF_PA);
      float* pb = at<float>(blk, BUF_PB);
      if ((rc = gemm(blk->w.w1, F, nullptr, 0, nullptr, 0, 1, D, xb, D / c.gx, c.gx, pa, F))) return rc;
      if ((rc = gemm(blk->w.w3, F, nullptr, 0, nullptr, 0, 1, D, xb, D / c.gx, c.gx, pb, F))) return rc;
      FfnMergeArgs m{};
      m.P1 = pa;
      m.P3 = pb;
      m.seg_stride = (int64_t)batch * F;
      m.nseg = c.gx;
      m.M = batch;
      m.N = F;
      m.quant = c.quant;
      m.act = ACT_SWIGLU;
      m.out_f32 = hbuf;
      m.out_bf16 = hb;
      m.bf16_split = 1;
      if ((rc = launch_ffn_merge(m, s))) return rc;
    }
    // a9
    if ((rc = stage_mark(blk, 5, s))) return rc;
    p2 = tc_split((int64_t)nseg2 * ((D + 127) / 128), F / nseg2, (int64_t)nseg2 * D, batch,
                  kW2MaxParts);
    if ((rc = gemm(blk->w.w2, D, nullptr, 0, nullptr, 0, 1, F, hb, F / nseg2 / p2, nseg2 * p2, part,
                   D)))
      return rc;
    if (phase == 1) return pack_step(blk, part, p2, batch, s);
  }
  // a10
  if ((rc = stage_mark(blk, 6, s))) return rc;
  if ((rc = merge_step(blk, x, part, nseg2, p2, batch, s, 1))) return rc;
  return stage_mark(blk, TP_BLOCK_STAGES, s);
}

// Batch 1-2, 1D partition: the whole block as one persistent kernel (*used set
// when it ran; otherwise the caller runs the kernel-per-step path).
int block_forward_persistent(tp_block* blk, float* x, void* kc, void* vc, const int32_t* pos,
                             int batch, cudaStream_t s, bool* used) {
  *used = false;
  const Cfg& c = blk->c;
  const tp_dims& d = c.d;
  const int D = d.dim, F = d.ffn_dim, QD = d.n_heads * d.head_dim, KD = d.n_kv_heads * d.head_dim;
  BpArgs a{};
  a.D = D;
  a.F = F;
  a.H = d.n_heads;
  a.Hkv = d.n_kv_heads;
  a.QD = QD;
  a.n = c.n;
  a.quant = c.quant;
  a.max_seq = d.max_seq;
  a.nb = batch;
  a.nchunk = c.nchunk;
  a.eps = d.norm_eps;
  a.theta = d.rope_theta;
  a.attn_norm = static_cast<const float*>(blk->w.attn_norm);
  a.ffn_norm = static_cast<const float*>(blk->w.ffn_norm);
  const auto wp = [](const void* p) { return static_cast<const uint16_t*>(p); };
  a.g[0] = BpGemv{{wp(blk->w.wq), wp(blk->w.wk), wp(blk->w.wv)}, {QD, KD, KD}, D, D, 1, QD + 2 * KD, 0, 0};
  a.g[1] = BpGemv{{wp(blk->w.wo), nullptr, nullptr}, {D, 0, 0}, QD, QD / c.n, c.n, D, 0, 0};
  a.g[2] = BpGemv{{wp(blk->w.w1), wp(blk->w.w3), nullptr}, {F, 0, 0}, D, D, 1, 2 * F, 0, 0};
  a.g[3] = BpGemv{{wp(blk->w.w2), nullptr, nullptr}, {D, 0, 0}, F, F / c.n, c.n, D, 0, 0};
  if (!plan_block_persistent(a, batch)) return TP_OK;
  a.x = x;
  a.kc = static_cast<uint16_t*>(kc);
  a.vc = static_cast<uint16_t*>(vc);
  a.pos = pos;
  a.xq = at<int8_t>(blk, BUF_XQ);
  a.xd = at<float>(blk, BUF_XD);
  a.xn = at<float>(blk, BUF_XN);
  a.q = at<float>(blk, BUF_Q);
  a.part_o = at<float>(blk, BUF_PO);
  a.part_ml = at<float>(blk, BUF_PML);
  a.att = at<float>(blk, BUF_ATT);
  a.part = at<float>(blk, BUF_PART);
  a.xmid = at<float>(blk, BUF_XMID);
  a.ssq = at<float>(blk, BUF_SSQ);
  a.h = at<float>(blk, BUF_H);
  a.err = at<int>(blk, BUF_ERR);
  a.bar = reinterpret_cast<unsigned*>(blk->ws + blk->L.off[BUF_ERR] + kCountersOff);
  a.trace = blk->trace;
  *used = true;
  return launch_block_persistent(a, batch, s);
}

// One block forward (the distributed-llama root-node order for one layer).
// chained: x was produced by the previous block's final merge of this same
// launch sequence, which left the row sums of squares in the workspace (inside
// a model); the final merge here leaves them for the next block.
// phase: -1 the whole step; 0 / 1 / 2 the three steps of a rank block (a1-a5 and
// the pack of its W_O partials; the merge of the gathered buffer, a7-a9 and the
// pack of its W2 partials; the final merge), between which the caller exchanges
// the sync buffers. seq (nullable): the cache sequence of each row, in caches of
// nseq sequences (rows of one sequence at consecutive positions: a prefill chunk).
int block_forward_impl(tp_block* blk, float* x, void* kc, void* vc, const int32_t* pos, int batch,
                       cudaStream_t s, bool chained = false, int phase = -1,
                       const int32_t* seq = nullptr, int nseq = 0) {
  if (!blk->bar_ready) {  // error word and counters start at zero (first use of the workspace)
    if (cudaMemsetAsync(blk->ws + blk->L.off[BUF_ERR], 0, blk->L.size[BUF_ERR], s) != cudaSuccess)
      return TP_ECUDA;
    blk->bar_ready = true;
  }
  // batched decode on the tensor cores (bf16 weights); int8 weights stay on the
  // weight-streaming kernels at every batch (2 rows per launch)
  if (batch >= kTcMinBatch && !blk->wq8)
    return block_forward_tc(blk, x, kc, vc, pos, batch, s, chained, phase, seq, nseq);
  if (batch <= 2 && blk->c.partition == TP_PART_1D && !blk->events && blk->persistent &&
      blk->c.world == 0 && !seq) {
    bool used = false;
    const int rc = block_forward_persistent(blk, x, kc, vc, pos, batch, s, &used);
    if (used || rc) return rc;
  }
  const Cfg& c = blk->c;
  const tp_dims& d = c.d;
  const int D = d.dim, F = d.ffn_dim, H = d.n_heads, Hkv = d.n_kv_heads, hd = d.head_dim;
  const int QD = H * hd;
  int rc;
  float* part = at<float>(blk, BUF_PART);
  float* hbuf = at<float>(blk, BUF_H);
  const int nseg2 = c.partition == TP_PART_1D ? c.n : c.gy;
  // context splits of the attention, which the W_O GEMV's staging combines
  const int att_nsplit = attention_nsplit(batch, H, Hkv, d.max_seq);

  if (phase <= 0) {
    // a1-a4: RMSNorm (+Q8, the buffer every slice reads) fused into the q/k/v slice
    // products, with RoPE and the cache write in the epilogue
    if ((rc = stage_mark(blk, 0, s))) return rc;
    {
      GemvArgs a{};
      a.w[0] = static_cast<const uint16_t*>(blk->w.wq);
      a.w[1] = static_cast<const uint16_t*>(blk->w.wk);
      a.w[2] = static_cast<const uint16_t*>(blk->w.wv);
      if (blk->wq8) {
        a.wd[0] = blk->wd_q;
        a.wd[1] = blk->wd_k;
        a.wd[2] = blk->wd_v;
      }
      a.rows[0] = QD;
      a.rows[1] = Hkv * hd;
      a.rows[2] = Hkv * hd;
      a.ldw = D;
      a.Ks = D;
      a.nseg = 1;
      set_norm_input(blk, a, x, blk->w.attn_norm);
      if (chained) {
        a.ssq = at<float>(blk, BUF_SSQ);
        a.ssq_parts = merge_ssq_parts(D);
      }
      a.nb = batch;
      a.qout = at<float>(blk, BUF_Q);
      a.kc = static_cast<uint16_t*>(kc);
      a.vc = static_cast<uint16_t*>(vc);
      a.pos = pos;
      a.seq = seq;
      a.n_heads = H;
      a.n_kv_heads = Hkv;
      a.max_seq = d.max_seq;
      a.theta = d.rope_theta;
      a.err = at<int>(blk, BUF_ERR);
      set_gemv_trace(blk, a, 0);
      if ((rc = launch_gemv(a, EPI_QKV, s))) return rc;
    }
    // a4: attention per head slice (context chunks, then their combination)
    if ((rc = stage_mark(blk, 1, s))) return rc;
    {
      AttnArgs a{};
      a.q = at<float>(blk, BUF_Q);
      a.kc = static_cast<const uint16_t*>(kc);
      a.vc = static_cast<const uint16_t*>(vc);
      a.pos = pos;
      a.seq = seq;
      a.nseq = nseq;
      a.B = batch;
      a.H = H;
      a.Hkv = Hkv;
      a.max_seq = d.max_seq;
      a.nchunk = c.nchunk;
      a.part_o = at<float>(blk, BUF_PO);
      a.part_ml = at<float>(blk, BUF_PML);
      a.att = at<float>(blk, BUF_ATT);
      a.nsplit = att_nsplit;
      a.err = at<int>(blk, BUF_ERR);
      if ((rc = launch_attention(a, s, false))) return rc;  // W_O's staging combines the splits
    }
    // a5: W_O row-split partials, one plane per slice
    if ((rc = stage_mark(blk, 2, s))) return rc;
    {
      GemvArgs a{};
      a.w[0] = static_cast<const uint16_t*>(blk->w.wo);
      if (blk->wq8) a.wd[0] = blk->wd_o;
      a.rows[0] = D;
      a.ldw = QD;
      a.Ks = QD / c.n;
      a.nseg = c.n;
      a.att_po = at<float>(blk, BUF_PO);
      a.att_pml = at<float>(blk, BUF_PML);
      a.att_nsplit = att_nsplit;
      a.att_out = at<float>(blk, BUF_ATT);
      a.pos = pos;
      a.n_heads = H;
      a.ldx = QD;
      a.nb = batch;
      a.out = part;
      a.out_seg = (int64_t)batch * D;
      a.ldo = D;
      a.err = at<int>(blk, BUF_ERR);
      set_gemv_trace(blk, a, 1);
      if ((rc = launch_gemv(a, EPI_PLAIN, s))) return rc;
    }
    if (phase == 0) return pack_step(blk, part, 1, batch, s);
  }
  if (phase <= 1) {
    // a6: sync + dequantise + merge into the residual (a rank block: of the
    // gathered buffer)
    if ((rc = stage_mark(blk, 3, s))) return rc;
    if ((rc = merge_step(blk, x, part, c.n, 1, batch, s, 0))) return rc;
    // a7-a8: RMSNorm (+Q8) fused into the W1/W3 slice products, SwiGLU epilogue
    if ((rc = stage_mark(blk, 4, s))) return rc;
    if (c.partition == TP_PART_1D) {
      GemvArgs a{};
      a.w[0] = static_cast<const uint16_t*>(blk->w.w1);
      a.w[1] = static_cast<const uint16_t*>(blk->w.w3);
      if (blk->wq8) {
        a.wd[0] = blk->wd_1;
        a.wd[1] = blk->wd_3;
      }
      a.rows[0] = F;
      a.ldw = D;
      a.Ks = D;
      a.nseg = 1;
      set_norm_input(blk, a, x, blk->w.ffn_norm);
      a.ssq = at<float>(blk, BUF_SSQ);  // written by the merge just above
      a.ssq_parts = merge_ssq_parts(D);
      a.nb = batch;
      a.out = hbuf;
      a.ldo = F;
      a.err = at<int>(blk, BUF_ERR);
      set_gemv_trace(blk, a, 2);
      if ((rc = launch_gemv(a, EPI_SWIGLU, s))) return rc;
    } else {
      // 2D stage 1: partials over the gx dim-slices for W1 and W3, merged with SwiGLU
      float* pa = at<float>(blk, BUF_PA);
      float* pb = at<float>(blk, BUF_PB);
      for (int m = 0; m < 2; ++m) {
        GemvArgs a{};
        a.w[0] = static_cast<const uint16_t*>(m == 0 ? blk->w.w1 : blk->w.w3);
        a.rows[0] = F;
        a.ldw = D;
        a.Ks = D / c.gx;
        a.nseg = c.gx;
        set_norm_input(blk, a, x, blk->w.ffn_norm);
        a.ssq = at<float>(blk, BUF_SSQ);
        a.ssq_parts = merge_ssq_parts(D);
        a.nb = batch;
        a.out = m == 0 ? pa : pb;
        a.out_seg = (int64_t)batch * F;
        a.ldo = F;
        a.err = at<int>(blk, BUF_ERR);
        if ((rc = launch_gemv(a, EPI_PLAIN, s))) return rc;
      }
      FfnMergeArgs m{};
      m.P1 = pa;
      m.P3 = pb;
      m.seg_stride = (int64_t)batch * F;
      m.nseg = c.gx;
      m.M = batch;
      m.N = F;
      m.quant = c.quant;
      m.act = ACT_SWIGLU;
      m.out_f32 = hbuf;
      if ((rc = launch_ffn_merge(m, s))) return rc;
    }
    // a9: W2 row-split partials
    if ((rc = stage_mark(blk, 5, s))) return rc;
    {
      GemvArgs a{};
      a.w[0] = static_cast<const uint16_t*>(blk->w.w2);
      if (blk->wq8) a.wd[0] = blk->wd_2;
      a.rows[0] = D;
      a.ldw = F;
      a.Ks = F / nseg2;
      a.nseg = nseg2;
      a.x = hbuf;
      a.ldx = F;
      a.nb = batch;
      a.out = part;
      a.out_seg = (int64_t)batch * D;
      a.ldo = D;
      a.err = at<int>(blk, BUF_ERR);
      set_gemv_trace(blk, a, 3);
      if ((rc = launch_gemv(a, EPI_PLAIN, s))) return rc;
    }
    if (phase == 1) return pack_step(blk, part, 1, batch, s);
  }
  // a10: sync + dequantise + merge
  if ((rc = stage_mark(blk, 6, s))) return rc;
  if ((rc = merge_step(blk, x, part, nseg2, 1, batch, s, 1))) return rc;
  return stage_mark(blk, TP_BLOCK_STAGES, s);
}

__global__ void k_embed(const uint16_t* __restrict__ emb, const int32_t* __restrict__ tok, int dim,
                        float* __restrict__ x) {
  pdl_launch_dependents();
  pdl_wait();
  const int b = blockIdx.x;
  const uint16_t* row = emb + (size_t)tok[b] * dim;
  for (int i = threadIdx.x; i < dim; i += blockDim.x)
    x[(size_t)b * dim + i] = __uint_as_float(((uint32_t)row[i]) << 16);
}

bool weights_aligned(const tp_block_weights* w) {
  return aligned16(w->attn_norm) && aligned16(w->wq) && aligned16(w->wk) && aligned16(w->wv) &&
         aligned16(w->wo) && aligned16(w->ffn_norm) && aligned16(w->w1) && aligned16(w->w3) &&
         aligned16(w->w2);
}

bool weights_present(const tp_block_weights* w) {
  return w && w->attn_norm && w->wq && w->wk && w->wv && w->wo && w->ffn_norm && w->w1 && w->w3 &&
         w->w2;
}

}  // namespace tp_api

using namespace tp_api;

extern "C" {

const char* tp_status_string(int st) {
  switch (st) {
    case TP_OK: return "ok";
    case TP_EINVAL: return "invalid argument";
    case TP_EWORKSPACE: return "workspace missing or too small";
    case TP_EARCH: return "device is not sm_100 (B200)";
    case TP_ECUDA: return "CUDA runtime error";
    case TP_ENOTSUP: return "not supported by this library";
    case TP_EALIGN: return "pointer not 16-byte aligned";
    case TP_ESCRATCH: return "workspace exceeds the fixed scratch of the no-allocation entry point";
    default: return "unknown status";
  }
}

const char* tp_version(void) { return "tp_block sm_100a 1"; }

int tp_block_workspace_bytes(const tp_dims* dims, int n_slices, int partition, int sync_quant,
                             size_t* out_bytes) {
  Cfg c;
  int rc = check_cfg(dims, n_slices, partition, sync_quant, &c);
  if (rc) return rc;
  if (!out_bytes) return TP_EINVAL;
  *out_bytes = block_layout(c).total;
  return TP_OK;
}

int tp_block_create(const tp_dims* dims, int n_slices, int partition, int sync_quant,
                    const tp_block_weights* w, void* workspace, size_t ws_bytes, tp_block** out) {
  if (!out) return TP_EINVAL;
  *out = nullptr;
  Cfg c;
  int rc = check_cfg(dims, n_slices, partition, sync_quant, &c);
  if (rc) return rc;
  if (!weights_present(w)) return TP_EINVAL;
  if (!weights_aligned(w)) return TP_EALIGN;
  Layout L = block_layout(c);
  if (!workspace || ws_bytes < L.total) return TP_EWORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255) != 0) return TP_EALIGN;
  rc = device_check();
  if (rc) return rc;
  tp_block* b = new (std::nothrow) tp_block;
  if (!b) return TP_EINVAL;
  b->c = c;
  b->L = L;
  b->w = *w;
  b->ws = static_cast<uint8_t*>(workspace);
  b->ws_bytes = ws_bytes;
  b->events = nullptr;
  b->bar_ready = false;
  b->trace = nullptr;
  b->persistent = persistent_default() ? 1 : 0;
  b->wq8 = false;
  b->phase_next = 0;
  b->phase_batch = 0;
  *out = b;
  return TP_OK;
}

int tp_block_rank_workspace_bytes(const tp_dims* dims, int n_slices, int sync_quant, int rank,
                                  int world, size_t* out_bytes) {
  Cfg c;
  const int rc = check_rank_cfg(dims, n_slices, sync_quant, rank, world, &c);
  if (rc) return rc;
  if (!out_bytes) return TP_EINVAL;
  *out_bytes = block_layout(c).total;
  return TP_OK;
}

int tp_block_create_rank(const tp_dims* dims, int n_slices, int sync_quant, int rank, int world,
                         const tp_block_weights* w, void* workspace, size_t ws_bytes,
                         tp_block** out) {
  if (!out) return TP_EINVAL;
  *out = nullptr;
  Cfg c;
  int rc = check_rank_cfg(dims, n_slices, sync_quant, rank, world, &c);
  if (rc) return rc;
  if (!weights_present(w)) return TP_EINVAL;
  if (!weights_aligned(w)) return TP_EALIGN;
  const Layout L = block_layout(c);
  if (!workspace || ws_bytes < L.total) return TP_EWORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255) != 0) return TP_EALIGN;
  rc = device_check();
  if (rc) return rc;
  tp_block* b = new (std::nothrow) tp_block;
  if (!b) return TP_EINVAL;
  b->c = c;
  b->L = L;
  b->w = *w;
  b->ws = static_cast<uint8_t*>(workspace);
  b->ws_bytes = ws_bytes;
  b->events = nullptr;
  b->bar_ready = false;
  b->trace = nullptr;
  b->persistent = 0;
  b->wq8 = false;
  b->phase_next = 0;
  b->phase_batch = 0;
  *out = b;
  return TP_OK;
}

int tp_block_rank_sync_bytes(const tp_block* blk, int batch, size_t* send_bytes) {
  if (!blk || !send_bytes || blk->c.world == 0) return TP_EINVAL;
  if (batch < 1 || batch > blk->c.d.max_batch) return TP_EINVAL;
  *send_bytes = (size_t)blk->c.n * (size_t)sync_slice_bytes(batch, blk->c.d.dim, blk->c.quant);
  return TP_OK;
}

int tp_block_rank_step(tp_block* blk, int phase, float* x, void* k_cache, void* v_cache,
                       const int32_t* pos, int batch, tp_stream stream) {
  if (!blk || blk->c.world == 0 || !x || !k_cache || !v_cache || !pos) return TP_EINVAL;
  if (batch < 1 || batch > blk->c.d.max_batch) return TP_EINVAL;
  if (phase != blk->phase_next || (phase > 0 && batch != blk->phase_batch)) return TP_EINVAL;
  if (!aligned16(x) || !aligned16(k_cache) || !aligned16(v_cache)) return TP_EALIGN;
  const int rc =
      block_forward_impl(blk, x, k_cache, v_cache, pos, batch, (cudaStream_t)stream, false, phase);
  blk->phase_next = rc ? 0 : (phase + 1) % 3;
  blk->phase_batch = batch;
  return rc;
}

int tp_block_create_q8w(const tp_dims* dims, int n_slices, int partition, int sync_quant,
                        const tp_block_weights_q8* w, void* workspace, size_t ws_bytes,
                        tp_block** out) {
  if (!out || !w || !dims) return TP_EINVAL;
  *out = nullptr;
  if (partition != TP_PART_1D || sync_quant != 1 || dims->ffn_dim % 64 != 0) return TP_EINVAL;
  const void* ptrs[] = {w->attn_norm, w->wq, w->wq_d, w->wk, w->wk_d, w->wv, w->wv_d, w->wo, w->wo_d,
                        w->ffn_norm, w->w1, w->w1_d, w->w3, w->w3_d, w->w2, w->w2_d};
  for (const void* p : ptrs) {
    if (!p) return TP_EINVAL;
    if (!aligned16(p)) return TP_EALIGN;
  }
  tp_block_weights codes{w->attn_norm, w->wq, w->wk, w->wv, w->wo, w->ffn_norm, w->w1, w->w3, w->w2};
  const int rc = tp_block_create(dims, n_slices, partition, sync_quant, &codes, workspace, ws_bytes, out);
  if (rc) return rc;
  tp_block* b = *out;
  b->wq8 = true;
  b->persistent = 0;
  b->wd_q = w->wq_d;
  b->wd_k = w->wk_d;
  b->wd_v = w->wv_d;
  b->wd_o = w->wo_d;
  b->wd_1 = w->w1_d;
  b->wd_3 = w->w3_d;
  b->wd_2 = w->w2_d;
  return TP_OK;
}

int tp_block_forward(tp_block* blk, float* x, void* k_cache, void* v_cache, const int32_t* pos,
                     int batch, tp_stream stream) {
  if (!blk || !x || !k_cache || !v_cache || !pos) return TP_EINVAL;
  if (blk->c.world > 0) return TP_EINVAL;  // a rank block runs through tp_block_rank_step
  if (batch < 1 || batch > blk->c.d.max_batch) return TP_EINVAL;
  if (!aligned16(x) || !aligned16(k_cache) || !aligned16(v_cache)) return TP_EALIGN;
  return block_forward_impl(blk, x, k_cache, v_cache, pos, batch, (cudaStream_t)stream);
}

int tp_block_forward_seq(tp_block* blk, float* x, void* k_cache, void* v_cache, const int32_t* pos,
                         const int32_t* seq, int n_seq, int batch, tp_stream stream) {
  if (!blk || !x || !k_cache || !v_cache || !pos || !seq || blk->c.world > 0) return TP_EINVAL;
  if (batch < 1 || n_seq < 1) return TP_EINVAL;
  if ((int64_t)n_seq * blk->c.d.n_kv_heads * blk->c.d.max_seq > INT32_MAX) return TP_EINVAL;
  if (!aligned16(x) || !aligned16(k_cache) || !aligned16(v_cache)) return TP_EALIGN;
  // more rows than max_batch: successive passes of max_batch rows in row order (each
  // pass's k/v are in the caches before the next pass's attention reads them)
  const int mb = blk->c.d.max_batch;
  for (int r0 = 0; r0 < batch; r0 += mb) {
    const int nb = batch - r0 < mb ? batch - r0 : mb;
    const int rc = block_forward_impl(blk, x + (size_t)r0 * blk->c.d.dim, k_cache, v_cache, pos + r0, nb,
                                      (cudaStream_t)stream, false, -1, seq + r0, n_seq);
    if (rc) return rc;
  }
  return TP_OK;
}

int tp_block_buffer(const tp_block* blk, int which, size_t* offset, size_t* bytes) {
  if (!blk || which < 0 || which >= BUF_COUNT) return TP_EINVAL;
  if (offset) *offset = blk->L.off[which];
  if (bytes) *bytes = blk->L.size[which];
  return TP_OK;
}

void tp_block_destroy(tp_block* blk) { delete blk; }

int tp_block_set_persistent(tp_block* blk, int enable) {
  if (!blk || (enable != 0 && enable != 1)) return TP_EINVAL;
  if (enable && blk->wq8) return TP_ENOTSUP;
  blk->persistent = enable;
  return TP_OK;
}

int tp_block_set_trace(tp_block* blk, void* trace, size_t bytes) {
  if (!blk) return TP_EINVAL;
  if (trace && bytes < (size_t)num_sms() * TP_BLOCK_TRACE_SLOTS * 8) return TP_EINVAL;
  blk->trace = static_cast<unsigned long long*>(trace);
  return TP_OK;
}

int tp_block_set_events(tp_block* blk, void* const* events, int n) {
  if (!blk) return TP_EINVAL;
  if (events && n != TP_BLOCK_STAGES + 1) return TP_EINVAL;
  blk->events = events;
  return TP_OK;
}

}  // extern "C"

namespace tp {
// Forward of one block over a caller-provided workspace using a handle that
// lives on the stack: no host or device allocation. Same checks as
// tp_block_create + tp_block_forward; the kernels' error word is zeroed on
// `stream` first (the workspace may hold an earlier call's contents).
int block_forward_on_workspace(const tp_dims* dims, int n_slices, int partition, int sync_quant,
                               const tp_block_weights* w, void* workspace, size_t ws_bytes,
                               float* x, void* k_cache, void* v_cache, const int32_t* pos,
                               int batch, cudaStream_t stream) {
  Cfg c;
  int rc = check_cfg(dims, n_slices, partition, sync_quant, &c);
  if (rc) return rc;
  if (!weights_present(w) || !x || !k_cache || !v_cache || !pos) return TP_EINVAL;
  if (!weights_aligned(w) || !aligned16(x) || !aligned16(k_cache) || !aligned16(v_cache))
    return TP_EALIGN;
  if (batch < 1 || batch > c.d.max_batch) return TP_EINVAL;
  tp_block blk;
  blk.c = c;
  blk.L = block_layout(c);
  if (!workspace || ws_bytes < blk.L.total) return TP_EWORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255) != 0) return TP_EALIGN;
  rc = device_check();
  if (rc) return rc;
  blk.w = *w;
  blk.ws = static_cast<uint8_t*>(workspace);
  blk.ws_bytes = ws_bytes;
  blk.events = nullptr;
  if (cudaMemsetAsync(blk.ws + blk.L.off[BUF_ERR], 0, blk.L.size[BUF_ERR], stream) != cudaSuccess)
    return TP_ECUDA;
  blk.bar_ready = true;  // the memset above covers every counter of BUF_ERR
  blk.trace = nullptr;
  blk.persistent = persistent_default() ? 1 : 0;
  blk.wq8 = false;
  blk.phase_next = 0;
  blk.phase_batch = 0;
  return block_forward_impl(&blk, x, k_cache, v_cache, pos, batch, stream);
}
}  // namespace tp

extern "C" {

// ------------------------------------------------------------------ model
int tp_model_workspace_bytes(const tp_dims* dims, int n_layers, int n_slices, int partition,
                             int sync_quant, size_t* out_bytes) {
  if (n_layers < 1 || !out_bytes) return TP_EINVAL;
  size_t blk = 0;
  int rc = tp_block_workspace_bytes(dims, n_slices, partition, sync_quant, &blk);
  if (rc) return rc;
  const size_t xb = align256((size_t)dims->max_batch * dims->dim * 4);
  *out_bytes = blk + 2 * xb;
  return TP_OK;
}

int tp_model_create(const tp_dims* dims, int n_layers, int n_slices, int partition, int sync_quant,
                    const tp_block_weights* layers, const void* embed, const float* final_norm,
                    const void* wcls, void* workspace, size_t ws_bytes, tp_model** out) {
  if (!out) return TP_EINVAL;
  *out = nullptr;
  size_t need = 0;
  int rc = tp_model_workspace_bytes(dims, n_layers, n_slices, partition, sync_quant, &need);
  if (rc) return rc;
  if (!layers || !embed || !final_norm || !wcls) return TP_EINVAL;
  if (dims->vocab <= 0 || dims->vocab % 2 != 0 || dims->vocab % n_slices != 0) return TP_EINVAL;
  if (!aligned16(embed) || !aligned16(final_norm) || !aligned16(wcls)) return TP_EALIGN;
  if (!workspace || ws_bytes < need) return TP_EWORKSPACE;
  size_t blk_bytes = 0;
  tp_block_workspace_bytes(dims, n_slices, partition, sync_quant, &blk_bytes);
  tp_model* m = new (std::nothrow) tp_model;
  if (!m) return TP_EINVAL;
  m->blocks = new (std::nothrow) tp_block[n_layers];
  if (!m->blocks) {
    delete m;
    return TP_EINVAL;
  }
  for (int l = 0; l < n_layers; ++l) {
    tp_block* bp = nullptr;
    rc = tp_block_create(dims, n_slices, partition, sync_quant, &layers[l], workspace, blk_bytes,
                         &bp);
    if (rc) {
      delete[] m->blocks;
      delete m;
      return rc;
    }
    m->blocks[l] = *bp;
    delete bp;
  }
  m->d = *dims;
  m->n_layers = n_layers;
  m->embed = embed;
  m->final_norm = final_norm;
  m->wcls = wcls;
  uint8_t* base = static_cast<uint8_t*>(workspace) + blk_bytes;
  m->x = reinterpret_cast<float*>(base);
  m->xnf = reinterpret_cast<float*>(base + align256((size_t)dims->max_batch * dims->dim * 4));
  *out = m;
  return TP_OK;
}

}  // extern "C"

namespace tp_api {
// The model step; seq (nullable) maps rows to the caches' nseq sequences.
int model_forward_impl(tp_model* m, const int32_t* tokens, void* k_cache, void* v_cache,
                       const int32_t* pos, const int32_t* seq, int nseq, int batch, float* logits,
                       cudaStream_t s) {
  const tp_dims& d = m->d;
  int rc0 = launch_pdl(k_embed, dim3(batch), dim3(256), 0, s,
                       static_cast<const uint16_t*>(m->embed), tokens, (int)d.dim, m->x);
  if (rc0) return rc0;
  const size_t layer_elems =
      (size_t)(seq ? nseq : d.max_batch) * d.n_kv_heads * (size_t)d.max_seq * d.head_dim;
  for (int l = 0; l < m->n_layers; ++l) {
    uint16_t* kc = static_cast<uint16_t*>(k_cache) + (size_t)l * layer_elems;
    uint16_t* vc = static_cast<uint16_t*>(v_cache) + (size_t)l * layer_elems;
    int rc = block_forward_impl(&m->blocks[l], m->x, kc, vc, pos, batch, s, l > 0, -1, seq, nseq);
    if (rc) return rc;
  }
  // RmsFinal(Norm) fused into the logits GEMV; the vocab column split writes each
  // slice's range of the output in place (the MergeLogits concatenation)
  GemvArgs a{};
  a.w[0] = static_cast<const uint16_t*>(m->wcls);
  a.rows[0] = d.vocab;
  a.ldw = d.dim;
  a.Ks = d.dim;
  a.nseg = 1;
  a.x = m->x;
  a.ldx = d.dim;
  a.gain = m->final_norm;
  a.eps = d.norm_eps;
  a.quant = 0;
  a.xn_out = m->xnf;
  a.nb = batch;
  a.out = logits;
  a.ldo = d.vocab;
  a.err = at<int>(&m->blocks[0], BUF_ERR);
  return launch_gemv(a, EPI_PLAIN, s);
}
}  // namespace tp_api

extern "C" {

int tp_model_forward(tp_model* m, const int32_t* tokens, void* k_cache, void* v_cache,
                     const int32_t* pos, int batch, float* logits, tp_stream stream) {
  if (!m || !tokens || !k_cache || !v_cache || !pos || !logits) return TP_EINVAL;
  if (batch < 1 || batch > m->d.max_batch) return TP_EINVAL;
  if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(logits)) return TP_EALIGN;
  return model_forward_impl(m, tokens, k_cache, v_cache, pos, nullptr, 0, batch, logits,
                            (cudaStream_t)stream);
}

int tp_model_forward_seq(tp_model* m, const int32_t* tokens, void* k_cache, void* v_cache,
                         const int32_t* pos, const int32_t* seq, int n_seq, int batch,
                         float* logits, tp_stream stream) {
  if (!m || !tokens || !k_cache || !v_cache || !pos || !seq || !logits) return TP_EINVAL;
  if (batch < 1 || n_seq < 1) return TP_EINVAL;
  if ((int64_t)n_seq * m->d.n_kv_heads * m->d.max_seq > INT32_MAX) return TP_EINVAL;
  if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(logits)) return TP_EALIGN;
  // more rows than max_batch: successive passes of max_batch rows through every layer,
  // in row order; each pass's logits rows start 16-byte aligned
  const int mb = m->d.max_batch;
  if (batch > mb && ((int64_t)mb * m->d.vocab) % 4 != 0) return TP_EALIGN;
  for (int r0 = 0; r0 < batch; r0 += mb) {
    const int nb = batch - r0 < mb ? batch - r0 : mb;
    const int rc = model_forward_impl(m, tokens + r0, k_cache, v_cache, pos + r0, seq + r0, n_seq, nb,
                                      logits + (size_t)r0 * m->d.vocab, (cudaStream_t)stream);
    if (rc) return rc;
  }
  return TP_OK;
}

int tp_model_set_persistent(tp_model* m, int enable) {
  if (!m || (enable != 0 && enable != 1)) return TP_EINVAL;
  for (int l = 0; l < m->n_layers; ++l) m->blocks[l].persistent = enable;
  return TP_OK;
}

void tp_model_destroy(tp_model* m) {
  if (!m) return;
  delete[] m->blocks;
  delete m;
}

// ------------------------------------------------------------------ Q8 codec
int tp_quantize_q8(const float* x, int8_t* q, float* d, int64_t n, tp_stream stream) {
  if (n < 0 || n % 32 != 0) return TP_EINVAL;
  if (n == 0) return TP_OK;
  if (!x || !q || !d) return TP_EINVAL;
  if (!aligned16(x) || !aligned16(q) || (reinterpret_cast<uintptr_t>(d) & 3)) return TP_EALIGN;
  int rc = device_check();
  if (rc) return rc;
  return launch_quantize(x, q, d, n, (cudaStream_t)stream);
}

int tp_dequantize_q8(const int8_t* q, const float* d, float* x, int64_t n, tp_stream stream) {
  if (n < 0 || n % 32 != 0) return TP_EINVAL;
  if (n == 0) return TP_OK;
  if (!x || !q || !d) return TP_EINVAL;
  if (!aligned16(x) || !aligned16(q) || (reinterpret_cast<uintptr_t>(d) & 3)) return TP_EALIGN;
  int rc = device_check();
  if (rc) return rc;
  return launch_dequantize(q, d, x, n, (cudaStream_t)stream);
}

}  // extern "C"
