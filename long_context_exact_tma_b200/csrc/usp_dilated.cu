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

namespace usp {

int dilated_fold_pair(const void* q, const void* k, const void* v, int B, int S, int Hq, int Hkv, int D, int causal,
                      int wp, int rp, float* o_run, float* lse_run, int* status, cudaStream_t st, int first) {
  if (first && rp != 1) return record_error(USP_ERR_INVALID_ARG, "only a pair with r = 1 covers every row");
  FwdLaunch L{};
  AttnGeom& g = L.g;
  g.B = B; g.S = S; g.Hq = Hq; g.Hkv = Hkv; g.D = D; g.causal = causal;
  g.P_u = g.P_r = g.P = g.n_ranks = 1;
  g.G = Hq / Hkv;
  g.Hq_l = Hq;
  g.Hkv_l = Hkv;
  L.status = status;
  L.wait_ns = current_wait_ns();
  L.step = -1;
  const unsigned long long tokq = 2ull * Hq * D, tokkv = 2ull * Hkv * D;  // bytes per token row
  const int n_seg = S / wp;
  // the offsets write disjoint heads of the running result: their (often small)
  // launches run side by side
  const int n_off = rp < Hq ? rp : Hq;
  const int n_st = n_off > 1 ? (n_off < kSideStreams ? n_off : kSideStreams) : 0;
  cudaStream_t side[kSideStreams];
  if (n_st) {
    const cudaError_t e = side_fork(st, n_st, side);
    if (e != cudaSuccess) return record_error(USP_ERR_CUDA, "side streams: %s", cudaGetErrorString(e));
  }
  int rc = USP_OK;
  for (int off = 0; off < n_off && rc == USP_OK; ++off) {
    const int kept = (wp - off + rp - 1) / rp;  // rows of a segment at offset off
    g.L = kept;
    g.c = kept;  // unused in the sub-problem mode
    FwdSub& sb = L.sub;
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
    sub_defaults(sb, Hkv);
    sb.first = first;
    rc = make_tmap_strided(&L.tm_q, static_cast<const uint8_t*>(q) + off * tokq, D, Hq, kept, sb.n_prob, rp * tokq,
                           wp * tokq);
    if (rc == USP_OK)
      rc = make_tmap_strided(&L.tm_k, static_cast<const uint8_t*>(k) + off * tokkv, D, Hkv, kept, sb.n_prob,
                             rp * tokkv, wp * tokkv);
    if (rc == USP_OK)
      rc = make_tmap_strided(&L.tm_v, static_cast<const uint8_t*>(v) + off * tokkv, D, Hkv, kept, sb.n_prob,
                             rp * tokkv, wp * tokkv);
    if (rc != USP_OK) break;
    const cudaError_t e = launch_attn_fwd(L, n_st ? side[off % n_st] : st);
    if (e != cudaSuccess) rc = record_error(USP_ERR_CUDA, "dilated attention launch: %s", cudaGetErrorString(e));
  }
  if (n_st) {
    const cudaError_t e = side_join(st, n_st);
    if (e != cudaSuccess && rc == USP_OK) rc = record_error(USP_ERR_CUDA, "side streams: %s", cudaGetErrorString(e));
  }
  return rc;
}

}  // namespace usp

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
  // A pair with r = 1 covers every row and head: run first, it writes the running
  // result, which then needs no initialisation (the log-sum-exp merge of the pairs
  // does not depend on their order).
  int p1 = -1;
  for (int p = 0; p < n_pairs && p1 < 0; ++p)
    if (r[p] == 1) p1 = p;
  cudaError_t e = cudaMemsetAsync(workspace, 0, sizeof(int), st);
  if (e == cudaSuccess && p1 < 0) e = usp::launch_fill_running(o_run, lse_run, rows, D, st);
  if (e != cudaSuccess) return record_error(USP_ERR_CUDA, "running-result init: %s", cudaGetErrorString(e));

  if (p1 >= 0) {
    const int rc = usp::dilated_fold_pair(q, k, v, B, S, Hq, Hkv, D, causal, w[p1], 1, o_run, lse_run,
                                          static_cast<int*>(workspace), st, 1);
    if (rc != USP_OK) return rc;
  }
  for (int p = 0; p < n_pairs; ++p) {
    if (p == p1) continue;
    const int rc = usp::dilated_fold_pair(q, k, v, B, S, Hq, Hkv, D, causal, w[p], r[p], o_run, lse_run,
                                          static_cast<int*>(workspace), st);
    if (rc != USP_OK) return rc;
  }
  e = usp::launch_lse_merge(o_run, lse_run, 1, rows, D, out, 0, lse, st);
  if (e != cudaSuccess) return record_error(USP_ERR_CUDA, "final merge launch: %s", cudaGetErrorString(e));
  return USP_OK;
}

// ---------------------------------------------------------------- backward
//
// The gradient of the pairs' combination: with the FINAL merged LSE and
// Delta_i = dO_i . O_i of every row, each pair contributes, at its kept rows,
// P_ij = exp(s_ij - LSE_i), dS_ij = P_ij (dO_i . V_j - Delta_i) -- the
// standard attention backward of that pair's sub-problems with the final
// LSE -- and the contributions of all pairs are summed. One launch of the
// key-major (dK, dV) and of the query-major (dQ) kernel per (pair, head
// offset), over the same strided tensor maps as the forward; dK and dV are
// accumulated in place (fp32), dQ in an fp32 workspace converted to bf16 last.
namespace {

using usp::record_error;

struct DilatedLaunchShape {
  int kept, n_seg, n_heads;
};

DilatedLaunchShape launch_shape(int S, int Hq, int w, int r, int off) {
  return DilatedLaunchShape{(w - off + r - 1) / r, S / w, (Hq - off + r - 1) / r};
}

}  // namespace

namespace usp {

// Floats of one row-table slot: the largest launch's n_prob * n_heads * Lp.
size_t slot_floats(int B, int S, int Hq, int w, int r) {
  size_t tbl = 0;
  for (int off = 0; off < r && off < Hq; ++off) {
    const DilatedLaunchShape sh = launch_shape(S, Hq, w, r, off);
    const size_t Lp = static_cast<size_t>((sh.kept + 127) / 128 * 128);
    const size_t n = static_cast<size_t>(B) * sh.n_seg * sh.n_heads * Lp;
    if (n > tbl) tbl = n;
  }
  return tbl;
}

size_t dilated_pair_table_floats(int B, int S, int Hq, int w, int r) {
  const int n_off = r < Hq ? r : Hq;  // launches of the pair, at most kSideStreams of them at a time
  return static_cast<size_t>(n_off < kSideStreams ? n_off : kSideStreams) * slot_floats(B, S, Hq, w, r);
}

int dilated_bwd_pair(const void* q, const void* k, const void* v, const void* dO, const float* lse,
                     const float* delta_all, float* dq_acc, float* dK, float* dV, float* lse2_t, float* delta_t, int B,
                     int S, int Hq, int Hkv, int D, int causal, int wp, int rp, int* status, cudaStream_t st,
                     int first) {
  if (first && rp != 1) return record_error(USP_ERR_INVALID_ARG, "only a pair with r = 1 covers every row");
  BwdLaunch L{};
  AttnGeom& g = L.g;
  g.B = B; g.S = S; g.Hq = Hq; g.Hkv = Hkv; g.D = D; g.causal = causal;
  g.P_u = g.P_r = g.P = g.n_ranks = 1;
  g.G = Hq / Hkv;
  g.Hq_l = Hq;
  g.Hkv_l = Hkv;
  L.status = status;
  L.wait_ns = current_wait_ns();
  L.lse2 = lse2_t;
  L.delta = delta_t;
  L.dk = dK;
  L.dv = dV;
  L.dq = nullptr;
  L.dq_acc = dq_acc;
  const unsigned long long tokq = 2ull * Hq * D, tokkv = 2ull * Hkv * D;
  // Offset o's launches write dQ, dK and dV only at the rows o + tau r of each
  // segment (whatever the kv heads they walk), so the offsets' writes are
  // disjoint: side streams, each with its own row-table slot.
  const int n_off = rp < Hq ? rp : Hq;
  const int n_st = n_off > 1 ? (n_off < kSideStreams ? n_off : kSideStreams) : 0;
  const size_t slot = slot_floats(B, S, Hq, wp, rp);
  cudaStream_t side[kSideStreams];
  if (n_st) {
    const cudaError_t e = side_fork(st, n_st, side);
    if (e != cudaSuccess) return record_error(USP_ERR_CUDA, "side streams: %s", cudaGetErrorString(e));
  }
  int rc = USP_OK;
  for (int off = 0; off < n_off && rc == USP_OK; ++off) {
    const DilatedLaunchShape sh = launch_shape(S, Hq, wp, rp, off);
    const int ks = n_st ? off % n_st : 0;  // stream and row-table slot
    cudaStream_t os = n_st ? side[ks] : st;
    L.lse2 = lse2_t + ks * slot;
    L.delta = delta_t + ks * slot;
    FwdSub& sb = L.sub;
    sb.active = 1;
    sb.n_prob = B * sh.n_seg;
    sb.L = sh.kept;
    sb.h0 = off;
    sb.h_step = rp;
    sb.n_heads = sh.n_heads;
    sb.n_seg = sh.n_seg;
    sb.w = wp;
    sb.off = off;
    sb.r = rp;
    sb.S = S;
    sb.Hq = Hq;
    sub_defaults(sb, Hkv);
    sb.first = first;  // write dQ, dK, dV instead of adding (r = 1 only: every row and head)
    if (rp % g.G == 0) {  // the offset's query heads o + j r sit in the kv heads o/G + j r/G, one each
      sb.kv0 = off / g.G;
      sb.kv_step = rp / g.G;
      sb.n_kv = sh.n_heads;
    }
    g.L = sh.kept;
    g.c = sh.kept;
    L.Lp = (sh.kept + 127) / 128 * 128;
    rc = make_tmap_strided(&L.tm_q, static_cast<const uint8_t*>(q) + off * tokq, D, Hq, sh.kept, sb.n_prob,
                           rp * tokq, wp * tokq);
    if (rc == USP_OK)
      rc = make_tmap_strided(&L.tm_do, static_cast<const uint8_t*>(dO) + off * tokq, D, Hq, sh.kept, sb.n_prob,
                             rp * tokq, wp * tokq);
    if (rc == USP_OK)
      rc = make_tmap_strided(&L.tm_k, static_cast<const uint8_t*>(k) + off * tokkv, D, Hkv, sh.kept, sb.n_prob,
                             rp * tokkv, wp * tokkv);
    if (rc == USP_OK)
      rc = make_tmap_strided(&L.tm_v, static_cast<const uint8_t*>(v) + off * tokkv, D, Hkv, sh.kept, sb.n_prob,
                             rp * tokkv, wp * tokkv);
    if (rc != USP_OK) break;
    cudaError_t e = launch_dilated_tables(lse, delta_all, lse2_t + ks * slot, delta_t + ks * slot, sb, L.Lp, os);
    if (e == cudaSuccess) e = launch_attn_bwd(L, os);
    if (e == cudaSuccess) e = launch_attn_bwd_dq(L, os);
    if (e != cudaSuccess) rc = record_error(USP_ERR_CUDA, "dilated backward launch: %s", cudaGetErrorString(e));
  }
  if (n_st) {
    const cudaError_t e = side_join(st, n_st);
    if (e != cudaSuccess && rc == USP_OK) rc = record_error(USP_ERR_CUDA, "side streams: %s", cudaGetErrorString(e));
  }
  return rc;
}

}  // namespace usp

namespace {

using usp::record_error;

size_t dilated_bwd_ws(int B, int S, int Hq, int D, int n_pairs, const int* w, const int* r, size_t* tbl_floats) {
  size_t tbl = 0;  // the largest per-launch table: n_prob * n_heads * Lp floats
  for (int p = 0; p < n_pairs; ++p) {
    const size_t n = usp::dilated_pair_table_floats(B, S, Hq, w[p], r[p]);
    if (n > tbl) tbl = n;
  }
  if (tbl_floats) *tbl_floats = tbl;
  const size_t rows = static_cast<size_t>(B) * S * Hq;
  // status | Delta of every row | fp32 dQ | two row tables
  return usp::kStatusBytes + rows * 4 + rows * D * 4 + 2 * tbl * 4;
}

int check_pairs(int S, int n_pairs, const int* w, const int* r) {
  if (!w || !r) return record_error(USP_ERR_INVALID_ARG, "null pair arrays");
  if (n_pairs < 1 || n_pairs > USP_DILATED_MAX_PAIRS)
    return record_error(USP_ERR_INVALID_ARG, "n_pairs must be 1..%d", USP_DILATED_MAX_PAIRS);
  for (int p = 0; p < n_pairs; ++p) {
    if (w[p] < 1 || r[p] < 1) return record_error(USP_ERR_INVALID_ARG, "pair %d: w and r must be positive", p);
    if (S % w[p] != 0) return record_error(USP_ERR_UNSUPPORTED, "pair %d: S (%d) is not a multiple of w (%d)", p, S, w[p]);
    if (r[p] > w[p]) return record_error(USP_ERR_UNSUPPORTED, "pair %d: r (%d) exceeds w (%d)", p, r[p], w[p]);
  }
  return USP_OK;
}

}  // namespace

extern "C" size_t usp_dilated_bwd_workspace_size(int B, int S, int Hq, int D, int n_pairs, const int* w,
                                                 const int* r) {
  if (B <= 0 || S <= 0 || Hq <= 0 || (D != 64 && D != 128)) return 0;
  if (!w || !r || n_pairs < 1 || n_pairs > USP_DILATED_MAX_PAIRS) return 0;
  for (int p = 0; p < n_pairs; ++p)
    if (w[p] < 1 || r[p] < 1 || r[p] > w[p] || S % w[p] != 0) return 0;
  return dilated_bwd_ws(B, S, Hq, D, n_pairs, w, r, nullptr);
}

extern "C" int usp_dilated_attn_bwd(const void* q, const void* k, const void* v, const void* out, const float* lse,
                                    const void* dO, void* dQ, float* dK, float* dV, int B, int S, int Hq, int Hkv,
                                    int D, int causal, int n_pairs, const int* w, const int* r, void* workspace,
                                    size_t ws_bytes, void* stream) {
  if (B <= 0 || S <= 0 || Hq <= 0 || Hkv <= 0) return record_error(USP_ERR_INVALID_ARG, "sizes must be positive");
  if (causal != 0 && causal != 1) return record_error(USP_ERR_INVALID_ARG, "causal must be 0 or 1");
  if (D != 64 && D != 128) return record_error(USP_ERR_UNSUPPORTED, "D must be 64 or 128 (got %d)", D);
  if (Hq % Hkv != 0) return record_error(USP_ERR_UNSUPPORTED, "Hq %% Hkv != 0");
  if (static_cast<long long>(B) * S * Hq >= (1LL << 31)) return record_error(USP_ERR_UNSUPPORTED, "too many rows");
  int rc = check_pairs(S, n_pairs, w, r);
  if (rc != USP_OK) return rc;
  if (!q || !k || !v || !out || !lse || !dO || !dQ || !dK || !dV)
    return record_error(USP_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse) || !aligned16(dO) ||
      !aligned16(dQ) || !aligned16(dK) || !aligned16(dV))
    return record_error(USP_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  size_t tbl = 0;
  const size_t need = dilated_bwd_ws(B, S, Hq, D, n_pairs, w, r, &tbl);
  if (!workspace || ws_bytes < need || !aligned16(workspace))
    return record_error(USP_ERR_WORKSPACE, "workspace needs %zu bytes (got %zu)", need, ws_bytes);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const long long rows = static_cast<long long>(B) * S * Hq;
  const long long kv_elems = static_cast<long long>(B) * S * Hkv * D;
  uint8_t* base = static_cast<uint8_t*>(workspace);
  float* delta_all = reinterpret_cast<float*>(base + usp::kStatusBytes);
  float* dq_acc = delta_all + rows;
  float* lse2_t = dq_acc + rows * D;
  float* delta_t = lse2_t + tbl;
  // As in the forward, a pair with r = 1 (every row and head) runs first and writes dQ's
  // accumulator, dK and dV, which then need no zeroing.
  int p1 = -1;
  for (int p = 0; p < n_pairs && p1 < 0; ++p)
    if (r[p] == 1) p1 = p;
  cudaError_t e = cudaMemsetAsync(workspace, 0, sizeof(int), st);
  if (p1 < 0) {
    if (e == cudaSuccess) e = cudaMemsetAsync(dq_acc, 0, rows * D * sizeof(float), st);
    if (e == cudaSuccess) e = cudaMemsetAsync(dK, 0, kv_elems * sizeof(float), st);
    if (e == cudaSuccess) e = cudaMemsetAsync(dV, 0, kv_elems * sizeof(float), st);
  }
  if (e == cudaSuccess) e = usp::launch_bwd_preprocess(out, dO, delta_all, rows, D, st);
  if (e != cudaSuccess) return record_error(USP_ERR_CUDA, "dilated backward init: %s", cudaGetErrorString(e));

  if (p1 >= 0) {
    rc = usp::dilated_bwd_pair(q, k, v, dO, lse, delta_all, dq_acc, dK, dV, lse2_t, delta_t, B, S, Hq, Hkv, D,
                               causal, w[p1], 1, static_cast<int*>(workspace), st, 1);
    if (rc != USP_OK) return rc;
  }
  for (int p = 0; p < n_pairs; ++p) {
    if (p == p1) continue;
    rc = usp::dilated_bwd_pair(q, k, v, dO, lse, delta_all, dq_acc, dK, dV, lse2_t, delta_t, B, S, Hq, Hkv, D,
                               causal, w[p], r[p], static_cast<int*>(workspace), st);
    if (rc != USP_OK) return rc;
  }
  e = usp::launch_f32_to_bf16(dq_acc, dQ, rows * D, st);
  if (e != cudaSuccess) return record_error(USP_ERR_CUDA, "dQ conversion: %s", cudaGetErrorString(e));
  return USP_OK;
}
