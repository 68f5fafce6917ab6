// usp_longnet.cu -- the per-rank compute of LongNet's distributed layout
// (LongNet slides, "LONGNET as a Distributed Trainer": a segment no longer than
// a device's slice is computed locally; a longer one has its key/value rows
// brought together by an all-gather and the local queries attend those global
// rows; in the backward the all-gather becomes a reduce-scatter).
//
// The sequence is split into contiguous slices of T tokens, one per rank. A
// dilated pair (w, r) with w <= T is the dilated attention of the rank's own
// segments (the launches of usp_dilated.cu on the slice). For w > T a segment
// spans G = w / T ranks; for head offset o the query heads o, o + r, ... keep
// the segment rows at positions = o (mod r), and each rank holds a contiguous
// run of them in kept order. The caller gathers every rank's kept K/V rows of
// those heads (only those: 1/r of the segment's rows, as LongNet sparsifies
// before it gathers) and this file's cross calls run the attention kernels in
// their sub-problem mode with a query window: the rank's kept query rows
// (kept indices k_lo ...) against all kept rows of the segment, the queries
// read in place through a tensor map with a row stride of r tokens and a head
// stride of r heads, the results folded at the rows' own positions and heads.
#include "../../include/usp.h"
#include "usp_internal.h"

namespace {

using usp::record_error;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Rows {
  int lp0, k_lo, n_rows, n_kept;
};

// This rank's share of the kept rows of offset o in its segment (rank g of G = w / T).
Rows rows_of(int T, int w, int r, int o, int g) {
  const long long a = static_cast<long long>(g) * T;  // segment position of the rank's first row
  const long long p0 = a + (((o - a) % r) + r) % r;    // first kept position at or after a
  Rows x;
  x.lp0 = static_cast<int>(p0 - a);
  x.k_lo = static_cast<int>((p0 - o) / r);
  x.n_rows = p0 < a + T ? static_cast<int>((a + T - p0 + r - 1) / r) : 0;
  x.n_kept = (w - o + r - 1) / r;
  return x;
}

int n_sel_of(int Hq, int r, int o) { return (Hq - o + r - 1) / r; }

int check_shape(int B, int T, int Hq, int Hkv, int D) {
  if (B <= 0 || T <= 0 || Hq <= 0 || Hkv <= 0) return record_error(USP_ERR_INVALID_ARG, "sizes must be positive");
  if (D != 64 && D != 128) return record_error(USP_ERR_UNSUPPORTED, "D must be 64 or 128 (got %d)", D);
  if (Hq % Hkv != 0) return record_error(USP_ERR_UNSUPPORTED, "Hq %% Hkv != 0");
  if (static_cast<long long>(B) * T * Hq >= (1LL << 31)) return record_error(USP_ERR_UNSUPPORTED, "too many rows");
  return USP_OK;
}

int check_local(int T, int w, int r) {
  if (w < 1 || r < 1 || r > w) return record_error(USP_ERR_INVALID_ARG, "need 1 <= r <= w (w=%d, r=%d)", w, r);
  if (w > T || T % w != 0)
    return record_error(USP_ERR_UNSUPPORTED, "a local pair needs w <= T and T %% w == 0 (T=%d, w=%d)", T, w);
  return USP_OK;
}

int check_cross(int T, int Hq, int w, int r, int o, int g) {
  if (w < 1 || r < 1 || r > w) return record_error(USP_ERR_INVALID_ARG, "need 1 <= r <= w (w=%d, r=%d)", w, r);
  if (w <= T || w % T != 0)
    return record_error(USP_ERR_UNSUPPORTED, "a gathered pair needs w > T and w %% T == 0 (T=%d, w=%d)", T, w);
  if (o < 0 || o >= r || o >= Hq) return record_error(USP_ERR_INVALID_ARG, "offset %d outside [0, min(r, Hq))", o);
  if (g < 0 || g >= w / T) return record_error(USP_ERR_INVALID_ARG, "rank %d outside its segment of %d", g, w / T);
  return USP_OK;
}

size_t fwd_ws(long long B, long long T, long long Hq, long long D) {
  return static_cast<size_t>(usp::kStatusBytes) + static_cast<size_t>(B * T * Hq) * (4 * D + 4);
}

// The largest row table of one offset's cross launch of a gathered pair (floats).
size_t cross_slot_floats(int B, int T, int Hq, int r) {
  size_t tbl = 0;
  for (int o = 0; o < r && o < Hq; ++o) {
    const size_t Lp = static_cast<size_t>(((T + r - 1) / r + 127) / 128 * 128);  // n_rows <= ceil(T / r)
    const size_t n = static_cast<size_t>(B) * n_sel_of(Hq, r, o) * Lp;
    if (n > tbl) tbl = n;
  }
  return tbl;
}

// The row tables a pair's launches on this rank need (floats): for a gathered
// pair one slot per head offset, up to usp::kSideStreams (offset o uses slot
// o mod kSideStreams, so the offsets' cross backwards may run concurrently).
size_t pair_table(int B, int T, int Hq, int w, int r) {
  if (w <= T) return usp::dilated_pair_table_floats(B, T, Hq, w, r);
  const int n_off = r < Hq ? r : Hq;
  const int slots = n_off < usp::kSideStreams ? n_off : usp::kSideStreams;
  return static_cast<size_t>(slots) * cross_slot_floats(B, T, Hq, r);
}

// Delta takes whole 16-byte groups, so the fp32 dQ after it stays aligned.
size_t delta_floats(size_t rows) { return (rows + 3) / 4 * 4; }

size_t bwd_ws(int B, int T, int Hq, int D, size_t tbl) {
  const size_t rows = static_cast<size_t>(B) * T * Hq;
  return usp::kStatusBytes + delta_floats(rows) * 4 + rows * D * 4 + 2 * tbl * 4;  // status | Delta | dQ | 2 tables
}

// The bwd workspace's parts; the tables take what follows dQ.
struct BwdParts {
  float *delta, *dq_acc, *lse2_t, *delta_t;
  size_t tbl;
};
BwdParts bwd_parts(void* ws, size_t ws_bytes, int B, int T, int Hq, int D) {
  const size_t rows = static_cast<size_t>(B) * T * Hq;
  BwdParts p{};
  uint8_t* base = static_cast<uint8_t*>(ws);
  p.delta = reinterpret_cast<float*>(base + usp::kStatusBytes);
  p.dq_acc = p.delta + delta_floats(rows);
  const size_t head = usp::kStatusBytes + delta_floats(rows) * 4 + rows * D * 4;
  p.tbl = ws_bytes > head ? (ws_bytes - head) / 8 / 4 * 4 : 0;
  p.lse2_t = p.dq_acc + rows * D;
  p.delta_t = p.lse2_t + p.tbl;
  return p;
}

// The sub-problem launch shape of a gathered (pair, offset) on this rank.
void cross_geometry(usp::AttnGeom& g, usp::FwdSub& sb, const Rows& x, int B, int T, int Hq, int D, int causal,
                    int r, int o, int n_sel) {
  g = usp::AttnGeom{};
  g.B = B; g.S = T; g.Hq = n_sel; g.Hkv = n_sel; g.D = D; g.causal = causal;
  g.P_u = g.P_r = g.P = g.n_ranks = 1;
  g.G = 1;
  g.Hq_l = n_sel;
  g.Hkv_l = n_sel;
  g.L = x.n_kept;
  g.c = x.n_kept;
  sb = usp::FwdSub{};
  sb.active = 1;
  sb.n_prob = B;  // one segment per sequence on this rank
  sb.L = x.n_kept;
  sb.h0 = 0;
  sb.h_step = 1;
  sb.n_heads = n_sel;
  sb.n_seg = 1;
  sb.w = T;
  sb.off = x.lp0;
  sb.r = r;
  sb.S = T;
  sb.Hq = Hq;
  sb.Lq = x.n_rows;
  sb.q_off = x.k_lo;
  sb.out_h0 = o;
  sb.out_hstep = r;
  sb.kS = x.n_kept;
  sb.kw = 0;
  sb.koff = 0;
  sb.kstep = 1;
  sb.kH = n_sel;
}

// Tensor maps of the rank's kept query-side rows (q or dO, read in place: row
// stride r tokens, head stride r heads, first row lp0, first head o) and of
// the compacted gathered rows [B][n_kept][n_sel][D].
int query_map(CUtensorMap* m, const void* x, const Rows& rw, int T, int Hq, int D, int r, int o, int n_sel, int B) {
  const unsigned long long tok = 2ull * Hq * D;
  return usp::make_tmap_strided_h(m, static_cast<const uint8_t*>(x) + rw.lp0 * tok + 2ull * o * D, D, n_sel,
                                  rw.n_rows, B, 2ull * r * D, r * tok, T * tok);
}
int gathered_map(CUtensorMap* m, const void* x, const Rows& rw, int D, int n_sel, int B) {
  const unsigned long long row = 2ull * n_sel * D;
  return usp::make_tmap_strided(m, x, D, n_sel, rw.n_kept, B, row, row * rw.n_kept);
}

}  // namespace

extern "C" {

int usp_longnet_rows(int T, int w, int r, int o, int g, int* lp0, int* k_lo, int* n_rows, int* n_kept) {
  if (T <= 0 || w < T || w % T != 0 || r < 1 || r > w || o < 0 || o >= r || g < 0 || g >= w / T)
    return record_error(USP_ERR_INVALID_ARG, "need w a multiple of T, 1 <= r <= w, 0 <= o < r, 0 <= g < w / T");
  const Rows x = rows_of(T, w, r, o, g);
  if (lp0) *lp0 = x.lp0;
  if (k_lo) *k_lo = x.k_lo;
  if (n_rows) *n_rows = x.n_rows;
  if (n_kept) *n_kept = x.n_kept;
  return USP_OK;
}

size_t usp_longnet_workspace_size(int B, int T, int Hq, int D, int n_pairs, const int* w, const int* r, int bwd) {
  if (B <= 0 || T <= 0 || Hq <= 0 || (D != 64 && D != 128)) return 0;
  if (!bwd) return fwd_ws(B, T, Hq, D);
  if (!w || !r || n_pairs < 1 || n_pairs > USP_DILATED_MAX_PAIRS) return 0;
  size_t tbl = 0;
  for (int p = 0; p < n_pairs; ++p) {
    if (w[p] < 1 || r[p] < 1 || r[p] > w[p]) return 0;
    if (w[p] <= T ? T % w[p] != 0 : w[p] % T != 0) return 0;
    const size_t n = pair_table(B, T, Hq, w[p], r[p]);
    if (n > tbl) tbl = n;
  }
  return bwd_ws(B, T, Hq, D, tbl);
}

int usp_longnet_fwd_begin(int B, int T, int Hq, int D, void* workspace, size_t ws_bytes, void* stream) {
  int rc = check_shape(B, T, Hq, Hq, D);
  if (rc != USP_OK) return rc;
  const size_t need = fwd_ws(B, T, Hq, D);
  if (!workspace || ws_bytes < need || !aligned16(workspace))
    return record_error(USP_ERR_WORKSPACE, "workspace needs %zu bytes (got %zu)", need, ws_bytes);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const long long rows = static_cast<long long>(B) * T * Hq;
  float* o_run = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + usp::kStatusBytes);
  cudaError_t e = cudaMemsetAsync(workspace, 0, sizeof(int), st);
  if (e == cudaSuccess) e = usp::launch_fill_running(o_run, o_run + rows * D, rows, D, st);
  return e == cudaSuccess ? USP_OK : record_error(USP_ERR_CUDA, "running-result init: %s", cudaGetErrorString(e));
}

int usp_longnet_fwd_local(const void* q, const void* k, const void* v, int B, int T, int Hq, int Hkv, int D,
                          int causal, int w, int r, void* workspace, size_t ws_bytes, void* stream) {
  int rc = check_shape(B, T, Hq, Hkv, D);
  if (rc == USP_OK) rc = check_local(T, w, r);
  if (rc != USP_OK) return rc;
  if (causal != 0 && causal != 1) return record_error(USP_ERR_INVALID_ARG, "causal must be 0 or 1");
  if (!q || !k || !v) return record_error(USP_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v))
    return record_error(USP_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  const size_t need = fwd_ws(B, T, Hq, D);
  if (!workspace || ws_bytes < need || !aligned16(workspace))
    return record_error(USP_ERR_WORKSPACE, "workspace needs %zu bytes (got %zu)", need, ws_bytes);
  const long long rows = static_cast<long long>(B) * T * Hq;
  float* o_run = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + usp::kStatusBytes);
  return usp::dilated_fold_pair(q, k, v, B, T, Hq, Hkv, D, causal, w, r, o_run, o_run + rows * D,
                                static_cast<int*>(workspace), static_cast<cudaStream_t>(stream));
}

int usp_longnet_fwd_cross(const void* q, const void* kc, const void* vc, int B, int T, int Hq, int Hkv, int D,
                          int causal, int w, int r, int o, int g, void* workspace, size_t ws_bytes, void* stream) {
  int rc = check_shape(B, T, Hq, Hkv, D);
  if (rc == USP_OK) rc = check_cross(T, Hq, w, r, o, g);
  if (rc != USP_OK) return rc;
  if (causal != 0 && causal != 1) return record_error(USP_ERR_INVALID_ARG, "causal must be 0 or 1");
  if (!q || !kc || !vc) return record_error(USP_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(kc) || !aligned16(vc))
    return record_error(USP_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  const size_t need = fwd_ws(B, T, Hq, D);
  if (!workspace || ws_bytes < need || !aligned16(workspace))
    return record_error(USP_ERR_WORKSPACE, "workspace needs %zu bytes (got %zu)", need, ws_bytes);
  const Rows x = rows_of(T, w, r, o, g);
  if (x.n_rows == 0) return USP_OK;  // no kept row of this offset on this rank
  const int n_sel = n_sel_of(Hq, r, o);
  const long long rows = static_cast<long long>(B) * T * Hq;
  usp::FwdLaunch L{};
  cross_geometry(L.g, L.sub, x, B, T, Hq, D, causal, r, o, n_sel);
  L.sub.o_run = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + usp::kStatusBytes);
  L.sub.lse_run = L.sub.o_run + rows * D;
  L.status = static_cast<int*>(workspace);
  L.wait_ns = usp::current_wait_ns();
  L.step = -1;
  rc = query_map(&L.tm_q, q, x, T, Hq, D, r, o, n_sel, B);
  if (rc == USP_OK) rc = gathered_map(&L.tm_k, kc, x, D, n_sel, B);
  if (rc == USP_OK) rc = gathered_map(&L.tm_v, vc, x, D, n_sel, B);
  if (rc != USP_OK) return rc;
  const cudaError_t e = usp::launch_attn_fwd(L, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? USP_OK : record_error(USP_ERR_CUDA, "cross attention launch: %s", cudaGetErrorString(e));
}

int usp_longnet_fwd_end(void* out, float* lse, int B, int T, int Hq, int D, void* workspace, size_t ws_bytes,
                        void* stream) {
  int rc = check_shape(B, T, Hq, Hq, D);
  if (rc != USP_OK) return rc;
  if (!out || !lse) return record_error(USP_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(out) || !aligned16(lse)) return record_error(USP_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  const size_t need = fwd_ws(B, T, Hq, D);
  if (!workspace || ws_bytes < need || !aligned16(workspace))
    return record_error(USP_ERR_WORKSPACE, "workspace needs %zu bytes (got %zu)", need, ws_bytes);
  const long long rows = static_cast<long long>(B) * T * Hq;
  float* o_run = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + usp::kStatusBytes);
  const cudaError_t e =
      usp::launch_lse_merge(o_run, o_run + rows * D, 1, rows, D, out, 0, lse, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? USP_OK : record_error(USP_ERR_CUDA, "final merge launch: %s", cudaGetErrorString(e));
}

int usp_longnet_bwd_begin(const void* out, const float* lse, const void* dO, float* dK, float* dV, int B, int T,
                          int Hq, int Hkv, int D, void* workspace, size_t ws_bytes, void* stream) {
  int rc = check_shape(B, T, Hq, Hkv, D);
  if (rc != USP_OK) return rc;
  if (!out || !lse || !dO || !dK || !dV) return record_error(USP_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(out) || !aligned16(lse) || !aligned16(dO) || !aligned16(dK) || !aligned16(dV))
    return record_error(USP_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  const size_t need = bwd_ws(B, T, Hq, D, 0);
  if (!workspace || ws_bytes < need || !aligned16(workspace))
    return record_error(USP_ERR_WORKSPACE, "workspace needs %zu bytes (got %zu)", need, ws_bytes);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const BwdParts p = bwd_parts(workspace, ws_bytes, B, T, Hq, D);
  const long long rows = static_cast<long long>(B) * T * Hq;
  const long long kv = static_cast<long long>(B) * T * Hkv * D;
  cudaError_t e = cudaMemsetAsync(workspace, 0, sizeof(int), st);
  if (e == cudaSuccess) e = cudaMemsetAsync(p.dq_acc, 0, rows * D * sizeof(float), st);
  if (e == cudaSuccess) e = cudaMemsetAsync(dK, 0, kv * sizeof(float), st);
  if (e == cudaSuccess) e = cudaMemsetAsync(dV, 0, kv * sizeof(float), st);
  if (e == cudaSuccess) e = usp::launch_bwd_preprocess(out, dO, p.delta, rows, D, st);
  return e == cudaSuccess ? USP_OK : record_error(USP_ERR_CUDA, "backward init: %s", cudaGetErrorString(e));
}

int usp_longnet_bwd_local(const void* q, const void* k, const void* v, const void* dO, const float* lse, float* dK,
                          float* dV, int B, int T, int Hq, int Hkv, int D, int causal, int w, int r, void* workspace,
                          size_t ws_bytes, void* stream) {
  int rc = check_shape(B, T, Hq, Hkv, D);
  if (rc == USP_OK) rc = check_local(T, w, r);
  if (rc != USP_OK) return rc;
  if (causal != 0 && causal != 1) return record_error(USP_ERR_INVALID_ARG, "causal must be 0 or 1");
  if (!q || !k || !v || !dO || !lse || !dK || !dV) return record_error(USP_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dO) || !aligned16(lse) || !aligned16(dK) ||
      !aligned16(dV))
    return record_error(USP_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  const size_t need = bwd_ws(B, T, Hq, D, pair_table(B, T, Hq, w, r));
  if (!workspace || ws_bytes < need || !aligned16(workspace))
    return record_error(USP_ERR_WORKSPACE, "workspace needs %zu bytes (got %zu)", need, ws_bytes);
  const BwdParts p = bwd_parts(workspace, ws_bytes, B, T, Hq, D);
  return usp::dilated_bwd_pair(q, k, v, dO, lse, p.delta, p.dq_acc, dK, dV, p.lse2_t, p.delta_t, B, T, Hq, Hkv, D,
                               causal, w, r, static_cast<int*>(workspace), static_cast<cudaStream_t>(stream));
}

int usp_longnet_bwd_cross(const void* q, const void* kc, const void* vc, const void* dO, const float* lse,
                          float* dkc, float* dvc, int B, int T, int Hq, int Hkv, int D, int causal, int w, int r,
                          int o, int g, void* workspace, size_t ws_bytes, void* stream) {
  int rc = check_shape(B, T, Hq, Hkv, D);
  if (rc == USP_OK) rc = check_cross(T, Hq, w, r, o, g);
  if (rc != USP_OK) return rc;
  if (causal != 0 && causal != 1) return record_error(USP_ERR_INVALID_ARG, "causal must be 0 or 1");
  if (!q || !kc || !vc || !dO || !lse || !dkc || !dvc) return record_error(USP_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(kc) || !aligned16(vc) || !aligned16(dO) || !aligned16(lse) || !aligned16(dkc) ||
      !aligned16(dvc))
    return record_error(USP_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  const size_t need = bwd_ws(B, T, Hq, D, pair_table(B, T, Hq, w, r));
  if (!workspace || ws_bytes < need || !aligned16(workspace))
    return record_error(USP_ERR_WORKSPACE, "workspace needs %zu bytes (got %zu)", need, ws_bytes);
  const Rows x = rows_of(T, w, r, o, g);
  const int n_sel = n_sel_of(Hq, r, o);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t grad = static_cast<size_t>(B) * x.n_kept * n_sel * D * sizeof(float);
  cudaError_t e = cudaMemsetAsync(dkc, 0, grad, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(dvc, 0, grad, st);
  if (e != cudaSuccess) return record_error(USP_ERR_CUDA, "gradient init: %s", cudaGetErrorString(e));
  if (x.n_rows == 0) return USP_OK;  // no query of this offset here: a zero contribution
  const BwdParts p = bwd_parts(workspace, ws_bytes, B, T, Hq, D);
  usp::BwdLaunch L{};
  cross_geometry(L.g, L.sub, x, B, T, Hq, D, causal, r, o, n_sel);
  L.status = static_cast<int*>(workspace);
  L.wait_ns = usp::current_wait_ns();
  L.Lp = (x.n_rows + 127) / 128 * 128;
  const size_t slot = static_cast<size_t>(o % usp::kSideStreams) * cross_slot_floats(B, T, Hq, r);
  float* const lse2_t = p.lse2_t + slot;  // this offset's row-table slot
  float* const delta_t = p.delta_t + slot;
  L.lse2 = lse2_t;
  L.delta = delta_t;
  L.dk = dkc;
  L.dv = dvc;
  L.dq = nullptr;
  L.dq_acc = p.dq_acc;
  rc = query_map(&L.tm_q, q, x, T, Hq, D, r, o, n_sel, B);
  if (rc == USP_OK) rc = query_map(&L.tm_do, dO, x, T, Hq, D, r, o, n_sel, B);
  if (rc == USP_OK) rc = gathered_map(&L.tm_k, kc, x, D, n_sel, B);
  if (rc == USP_OK) rc = gathered_map(&L.tm_v, vc, x, D, n_sel, B);
  if (rc != USP_OK) return rc;
  e = usp::launch_dilated_tables(lse, p.delta, lse2_t, delta_t, L.sub, L.Lp, st);
  if (e == cudaSuccess) e = usp::launch_attn_bwd(L, st);
  if (e == cudaSuccess) e = usp::launch_attn_bwd_dq(L, st);
  return e == cudaSuccess ? USP_OK : record_error(USP_ERR_CUDA, "cross backward launch: %s", cudaGetErrorString(e));
}

int usp_longnet_bwd_end(void* dQ, int B, int T, int Hq, int D, void* workspace, size_t ws_bytes, void* stream) {
  int rc = check_shape(B, T, Hq, Hq, D);
  if (rc != USP_OK) return rc;
  if (!dQ || !aligned16(dQ)) return record_error(USP_ERR_INVALID_ARG, "dQ must be a 16-byte aligned pointer");
  const size_t need = bwd_ws(B, T, Hq, D, 0);
  if (!workspace || ws_bytes < need || !aligned16(workspace))
    return record_error(USP_ERR_WORKSPACE, "workspace needs %zu bytes (got %zu)", need, ws_bytes);
  const BwdParts p = bwd_parts(workspace, ws_bytes, B, T, Hq, D);
  const long long rows = static_cast<long long>(B) * T * Hq;
  const cudaError_t e = usp::launch_f32_to_bf16(p.dq_acc, dQ, rows * D, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? USP_OK : record_error(USP_ERR_CUDA, "dQ conversion: %s", cudaGetErrorString(e));
}

}  // extern "C"
