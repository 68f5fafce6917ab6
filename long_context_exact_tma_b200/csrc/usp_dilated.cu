// usp_dilated.cu -- LongNet dilated attention (forward) on the blockwise
// attention kernel of usp_attn_fwd.cu, in its sub-problem mode.
//
// What it computes (LongNet slides, "Abstract": dilated attention as a drop-in
// replacement for standard attention; "Results": segment lengths w and
// dilation ratios r, e.g. w = {2048, ..., 32768}, r = {1, 2, 4, 6, 12}): for
// each (w, r) pair the sequence is cut into segments of w tokens, every r-th
// row of a segment is kept starting at the offset h mod r of the query head h,
// and dense softmax attention runs among the kept rows of each segment (causal
// within it when asked). The pairs' results are combined with weights
// proportional to their softmax denominators, i.e. merged by log-sum-exp.
//
// On B200 nothing is gathered: for a pair (w, r) and an offset o the TMA
// tensor maps view Q, K and V as {D, heads, kept rows, segments} with a row
// stride of r token rows and a base o rows in, so the kernel's 128-row tiles
// ARE the kept rows of a segment. One launch per (pair, offset) covers the
// heads with that offset; its epilogue folds the result into a running fp32
// (O, LSE) in the workspace, and a last merge pass writes O (bf16) and LSE.
#include "../../include/usp.h"
#include "usp_internal.h"

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t dilated_ws(long long B, long long S, long long Hq, long long D) {
  return static_cast<size_t>(usp::kStatusBytes) + static_cast<size_t>(B * S * Hq) * (4 * D + 4);
}

}  // namespace

extern "C" size_t usp_dilated_workspace_size(int B, int S, int Hq, int D) {
  if (B <= 0 || S <= 0 || Hq <= 0 || (D != 64 && D != 128)) return 0;
  return dilated_ws(B, S, Hq, D);
}

extern "C" int usp_dilated_attn_fwd(const void* q, const void* k, const void* v, void* out, float* lse, int B,
                                    int S, int Hq, int Hkv, int D, int causal, int n_pairs, const int* w,
                                    const int* r, void* workspace, size_t ws_bytes, void* stream) {
  using usp::record_error;
  if (B <= 0 || S <= 0 || Hq <= 0 || Hkv <= 0) return record_error(USP_ERR_INVALID_ARG, "sizes must be positive");
  if (causal != 0 && causal != 1) return record_error(USP_ERR_INVALID_ARG, "causal must be 0 or 1");
  if (D != 64 && D != 128) return record_error(USP_ERR_UNSUPPORTED, "D must be 64 or 128 (got %d)", D);
  if (Hq % Hkv != 0) return record_error(USP_ERR_UNSUPPORTED, "Hq %% Hkv != 0");
  if (static_cast<long long>(B) * S * Hq >= (1LL << 31)) return record_error(USP_ERR_UNSUPPORTED, "too many rows");
  if (!q || !k || !v || !out || !lse || !w || !r) return record_error(USP_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse))
    return record_error(USP_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  if (n_pairs < 1 || n_pairs > USP_DILATED_MAX_PAIRS)
    return record_error(USP_ERR_INVALID_ARG, "n_pairs must be 1..%d", USP_DILATED_MAX_PAIRS);
  for (int p = 0; p < n_pairs; ++p) {
    if (w[p] < 1 || r[p] < 1) return record_error(USP_ERR_INVALID_ARG, "pair %d: w and r must be positive", p);
    if (S % w[p] != 0) return record_error(USP_ERR_UNSUPPORTED, "pair %d: S (%d) is not a multiple of w (%d)", p, S, w[p]);
    if (r[p] > w[p]) return record_error(USP_ERR_UNSUPPORTED, "pair %d: r (%d) exceeds w (%d)", p, r[p], w[p]);
  }
  const size_t need = dilated_ws(B, S, Hq, D);
  if (!workspace || ws_bytes < need || !aligned16(workspace))
    return record_error(USP_ERR_WORKSPACE, "workspace needs %zu bytes (got %zu)", need, ws_bytes);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const long long rows = static_cast<long long>(B) * S * Hq;
  float* o_run = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + usp::kStatusBytes);
  float* lse_run = o_run + rows * D;
  cudaError_t e = cudaMemsetAsync(workspace, 0, sizeof(int), st);
  if (e == cudaSuccess) e = usp::launch_fill_running(o_run, lse_run, rows, D, st);
  if (e != cudaSuccess) return record_error(USP_ERR_CUDA, "running-result init: %s", cudaGetErrorString(e));

  usp::FwdLaunch L{};
  usp::AttnGeom& g = L.g;
  g.B = B; g.S = S; g.Hq = Hq; g.Hkv = Hkv; g.D = D; g.causal = causal;
  g.P_u = g.P_r = g.P = g.n_ranks = 1;
  g.G = Hq / Hkv;
  g.Hq_l = Hq;
  g.Hkv_l = Hkv;
  L.status = static_cast<int*>(workspace);
  L.wait_ns = usp::current_wait_ns();
  L.step = -1;
  const unsigned long long tokq = 2ull * Hq * D, tokkv = 2ull * Hkv * D;  // bytes per token row
  for (int p = 0; p < n_pairs; ++p) {
    const int wp = w[p], rp = r[p];
    const int n_seg = S / wp;
    for (int off = 0; off < rp && off < Hq; ++off) {
      const int kept = (wp - off + rp - 1) / rp;  // rows of a segment at offset off
      g.L = kept;
      g.c = kept;  // unused in the sub-problem mode
      usp::FwdSub& sb = L.sub;
      sb.active = 1;
      sb.n_prob = B * n_seg;
      sb.L = kept;
      sb.h0 = off;
      sb.h_step = rp;
      sb.n_heads = (Hq - off + rp - 1) / rp;
      sb.n_seg = n_seg;
      sb.w = wp;
      sb.off = off;
      sb.r = rp;
      sb.S = S;
      sb.Hq = Hq;
      sb.o_run = o_run;
      sb.lse_run = lse_run;
      int rc = usp::make_tmap_strided(&L.tm_q, static_cast<const uint8_t*>(q) + off * tokq, D, Hq, kept,
                                      sb.n_prob, rp * tokq, wp * tokq);
      if (rc == USP_OK)
        rc = usp::make_tmap_strided(&L.tm_k, static_cast<const uint8_t*>(k) + off * tokkv, D, Hkv, kept,
                                    sb.n_prob, rp * tokkv, wp * tokkv);
      if (rc == USP_OK)
        rc = usp::make_tmap_strided(&L.tm_v, static_cast<const uint8_t*>(v) + off * tokkv, D, Hkv, kept,
                                    sb.n_prob, rp * tokkv, wp * tokkv);
      if (rc != USP_OK) return rc;
      e = usp::launch_attn_fwd(L, st);
      if (e != cudaSuccess) return record_error(USP_ERR_CUDA, "dilated attention launch: %s", cudaGetErrorString(e));
    }
  }
  e = usp::launch_lse_merge(o_run, lse_run, 1, rows, D, out, 0, lse, st);
  if (e != cudaSuccess) return record_error(USP_ERR_CUDA, "final merge launch: %s", cudaGetErrorString(e));
  return USP_OK;
}
