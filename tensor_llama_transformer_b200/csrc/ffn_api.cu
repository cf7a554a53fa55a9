// tp_ffn_forward: the partitioned feed-forward layer.
//
// aiterms.tw "Tensor Parallelism", how it works: X replicated; Linear1 split by
// columns (each slice computes its own columns of the hidden layer, no
// communication); the activation applied locally; Linear2 split by rows (each
// slice produces a partial of the full output); one all-reduce. Pope et al.
// (CS349E lecture script, demo1_1d_vs_2d): 1D splits F only, 2D
// weight-stationary splits E over grid_x and F over grid_y, which adds a
// partial-sum stage before the activation.
//
// On one GPU every slice is a segment of the same launch: a segment is the
// contraction range one slice owns. TP_MERGE_FAITHFUL forms every slice's
// partial product on its own (float32) and sums the partials in slice order,
// each through the Q8 round trip when quantising: for bf16 inside the tensor-core
// GEMM (the CTA that owns an output tile computes its segments one after another
// and adds them up in its epilogue; in 1D the first stage has one segment, so its
// activation is applied to the accumulator directly), for float32 (and the 2D
// SwiGLU first stage) by writing each partial to its own plane of the workspace
// and summing the planes in the merge kernel. The sums are the same float32
// additions either way. With TP_MERGE_FUSED the slices' contraction ranges are
// accumulated in slice order inside the tensor-core accumulator instead, which
// is the sum of the exact partials rounded once.
#include "ffn.cuh"
#include "gemm_tc.cuh"

namespace tp {
namespace {

size_t a256(size_t v) { return (v + 255) & ~(size_t)255; }

struct FfnPlan {
  int nseg1, nseg2, Ks1, Ks2, swiglu, esize;
  bool planes1, planes2;  // stage 1 / stage 2 partials materialised in the workspace
  size_t off_err, off_p1a, off_p1b, off_h, off_p2, total;
};

int plan_ffn(const tp_ffn_desc* d, FfnPlan* p) {
  if (!d || !p) return TP_EINVAL;
  if (d->batch < 1 || d->E <= 0 || d->F <= 0) return TP_EINVAL;
  if (d->dtype != TP_F32 && d->dtype != TP_BF16) return TP_EINVAL;
  if (d->act != TP_ACT_RELU && d->act != TP_ACT_SWIGLU) return TP_EINVAL;
  if (d->sync_quant != 0 && d->sync_quant != 1) return TP_EINVAL;
  if (d->merge != TP_MERGE_FAITHFUL && d->merge != TP_MERGE_FUSED) return TP_EINVAL;
  if (d->E % 32 != 0 || d->F % 32 != 0) return TP_EINVAL;
  if (d->partition == TP_PART_1D) {
    if (d->n_slices < 1 || d->F % (32 * d->n_slices) != 0) return TP_EINVAL;
    p->nseg1 = 1;
    p->nseg2 = d->n_slices;
  } else if (d->partition == TP_PART_2D) {
    if (d->grid_x < 1 || d->grid_y < 1) return TP_EINVAL;
    if (d->E % (32 * d->grid_x) != 0 || d->F % (32 * d->grid_y) != 0) return TP_EINVAL;
    p->nseg1 = d->grid_x;
    p->nseg2 = d->grid_y;
  } else {
    return TP_EINVAL;
  }
  p->Ks1 = d->E / p->nseg1;
  p->Ks2 = d->F / p->nseg2;
  p->swiglu = d->act == TP_ACT_SWIGLU;
  p->esize = d->dtype == TP_F32 ? 4 : 2;
  if (d->merge == TP_MERGE_FUSED && (d->dtype != TP_BF16 || d->sync_quant)) return TP_ENOTSUP;
  const size_t B = d->batch, E = d->E, F = d->F;
  const bool fused = d->merge == TP_MERGE_FUSED;
  const bool f32 = d->dtype == TP_F32;
  // bf16: the tensor-core GEMM sums the segments itself, except for the 2D SwiGLU
  // first stage (two products per hidden value)
  p->planes1 = !fused && (f32 || (p->nseg1 > 1 && p->swiglu));
  p->planes2 = !fused && f32;
  size_t o = 0;
  p->off_err = o;
  o += 256;
  p->off_p1a = o;
  if (p->planes1) o += a256((size_t)p->nseg1 * B * F * 4);
  p->off_p1b = o;
  if (p->planes1 && p->swiglu) o += a256((size_t)p->nseg1 * B * F * 4);
  p->off_h = o;
  o += a256(B * F * p->esize);
  p->off_p2 = o;
  if (p->planes2) o += a256((size_t)p->nseg2 * B * E * 4);
  p->total = o;
  return TP_OK;
}

}  // namespace
}  // namespace tp

using namespace tp;

extern "C" {

int tp_ffn_workspace_bytes(const tp_ffn_desc* d, size_t* out_bytes) {
  FfnPlan p;
  int rc = plan_ffn(d, &p);
  if (rc) return rc;
  if (!out_bytes) return TP_EINVAL;
  *out_bytes = p.total;
  return TP_OK;
}

int tp_ffn_forward(const tp_ffn_desc* d, const void* X, const void* W1, const void* W3,
                   const void* W2, float* Y, void* workspace, size_t ws_bytes, tp_stream stream) {
  FfnPlan p;
  int rc = plan_ffn(d, &p);
  if (rc) return rc;
  if (!X || !W1 || !W2 || !Y || (p.swiglu && !W3)) return TP_EINVAL;
  if (!aligned16(X) || !aligned16(W1) || !aligned16(W2) || !aligned16(Y) ||
      (W3 && !aligned16(W3)))
    return TP_EALIGN;
  if (p.total > 0 && (!workspace || ws_bytes < p.total)) return TP_EWORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255) != 0) return TP_EALIGN;
  rc = device_check();
  if (rc) return rc;
  cudaStream_t s = (cudaStream_t)stream;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int B = d->batch, E = d->E, F = d->F;
  void* H = ws + p.off_h;
  int* err = reinterpret_cast<int*>(ws + p.off_err);

  if (d->merge == TP_MERGE_FUSED) {
    // stage 1: H = act(X W1^T [, X W3^T]) over the full E (slice order = K order)
    TcGemm g{};
    g.A[0] = X;
    g.Am[0] = B;
    g.nA = 1;
    g.lda = E;
    g.B = W1;
    g.ldb = E;
    g.B2 = p.swiglu ? W3 : nullptr;
    g.N = F;
    g.K = E;
    g.nseg = 1;
    g.epi = p.swiglu ? TC_EPI_SWIGLU_BF16 : TC_EPI_RELU_BF16;
    g.out = H;
    g.ldo = F;
    g.err = err;
    g.indep = TC_INDEP_B;  // the weights
    rc = launch_tc_gemm(g, s);
    if (rc) return rc;
    // stage 2: Y = H W2^T over the full F
    TcGemm g2{};
    g2.A[0] = H;
    g2.Am[0] = B;
    g2.nA = 1;
    g2.lda = F;
    g2.B = W2;
    g2.ldb = F;
    g2.N = E;
    g2.K = F;
    g2.nseg = 1;
    g2.epi = TC_EPI_STORE_F32;
    g2.out = Y;
    g2.ldo = E;
    g2.err = err;
    g2.indep = TC_INDEP_B;
    return launch_tc_gemm(g2, s);
  }

  float* P1a = reinterpret_cast<float*>(ws + p.off_p1a);
  float* P1b = reinterpret_cast<float*>(ws + p.off_p1b);
  float* P2 = reinterpret_cast<float*>(ws + p.off_p2);
  // one bf16 tensor-core product over nseg segments of Ks with epilogue `epi`
  auto tc = [&](const void* A, int64_t lda, const void* Bm, const void* Bm2, int64_t ldb, void* out,
                int M, int N, int Ks, int nseg, int epi, int quant) -> int {
    TcGemm g{};
    g.A[0] = A;
    g.Am[0] = M;
    g.nA = 1;
    g.lda = lda;
    g.B = Bm;
    g.B2 = Bm2;
    g.ldb = ldb;
    g.N = N;
    g.K = Ks;
    g.nseg = nseg;
    g.epi = epi;
    g.quant = quant;
    g.out = out;
    g.ldo = N;
    g.out_seg = (int64_t)M * N;
    g.err = err;
    g.indep = TC_INDEP_B;  // the weights
    return launch_tc_gemm(g, s);
  };
  // the partials of A B^T over nseg segments of Ks, one float32 plane each
  auto contract = [&](const void* A, int64_t lda, const void* Bm, int64_t ldb, float* P, int M,
                      int N, int Ks, int nseg) -> int {
    if (d->dtype == TP_F32) return launch_gemm_simt(TP_F32, A, lda, Bm, ldb, P, M, N, Ks, nseg, s);
    return tc(A, lda, Bm, nullptr, ldb, P, M, N, Ks, nseg, TC_EPI_STORE_F32, 0);
  };
  // in 1D the hidden columns stay local to their slice: no sync buffer there
  const int quant1 = d->partition == TP_PART_2D ? d->sync_quant : 0;

  // stage 1: H = act(sum over the E-segments of X W1^T [, X W3^T]) (one segment in 1D)
  if (!p.planes1) {
    if (p.nseg1 == 1)
      rc = tc(X, E, W1, p.swiglu ? W3 : nullptr, E, H, B, F, p.Ks1, 1,
              p.swiglu ? TC_EPI_SWIGLU_BF16 : TC_EPI_RELU_BF16, 0);
    else
      rc = tc(X, E, W1, nullptr, E, H, B, F, p.Ks1, p.nseg1, TC_EPI_SEGSUM_RELU_BF16, quant1);
    if (rc) return rc;
  } else {
    rc = contract(X, E, W1, E, P1a, B, F, p.Ks1, p.nseg1);
    if (rc) return rc;
    if (p.swiglu) {
      rc = contract(X, E, W3, E, P1b, B, F, p.Ks1, p.nseg1);
      if (rc) return rc;
    }
    FfnMergeArgs m{};
    m.P1 = P1a;
    m.P3 = p.swiglu ? P1b : nullptr;
    m.seg_stride = (int64_t)B * F;
    m.nseg = p.nseg1;
    m.M = B;
    m.N = F;
    m.quant = quant1;
    m.act = p.swiglu ? ACT_SWIGLU : ACT_RELU;
    if (d->dtype == TP_F32)
      m.out_f32 = static_cast<float*>(H);
    else
      m.out_bf16 = static_cast<uint16_t*>(H);
    rc = launch_ffn_merge(m, s);
    if (rc) return rc;
  }
  // stage 2: Y = sum over the F-segments of H W2^T
  if (!p.planes2) return tc(H, F, W2, nullptr, F, Y, B, E, p.Ks2, p.nseg2, TC_EPI_SEGSUM_F32,
                            d->sync_quant);
  rc = contract(H, F, W2, F, P2, B, E, p.Ks2, p.nseg2);
  if (rc) return rc;
  FfnMergeArgs m{};
  m.P1 = P2;
  m.seg_stride = (int64_t)B * E;
  m.nseg = p.nseg2;
  m.M = B;
  m.N = E;
  m.quant = d->sync_quant;
  m.act = ACT_NONE;
  m.out_f32 = Y;
  return launch_ffn_merge(m, s);
}

}  // extern "C"
