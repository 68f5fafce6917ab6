// usp_ring.cu -- the per-rank compute of a REAL multi-GPU USP mesh: one process
// per GPU holds one rank (ring index i, Ulysses index u) and runs, per ring
// step, its own queries against the one KV block it holds ("Boosting Spec
// Eagle", "The Solution": each ring device holds a slice of the sequence and
// passes key/value blocks to its neighbour; DeepSpeed-Ulysses summary, "Wie
// DeepSpeed-Ulysses funktioniert": the all-to-all before and after attention).
//
// These calls are the compute between the collectives; the collectives
// themselves (the Ulysses all-to-all inside a group, the ring send/receive of
// K/V and of the travelling dK/dV) are NCCL calls the caller makes. The
// attention kernels are those of the one-GPU emulation in their local mode:
// same tiles, same zigzag positions, but the rank's own buffers.
#include <string.h>

#include "../../include/usp.h"
#include "usp_internal.h"

namespace {

using usp::record_error;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int elem_size(int dtype) { return dtype == USP_BF16 ? 2 : dtype == USP_F32 ? 4 : 0; }

size_t local_rows(const usp::AttnGeom& g) { return static_cast<size_t>(g.B) * g.L * g.Hq_l; }
int padded(const usp::AttnGeom& g) { return (g.L + 127) / 128 * 128; }
size_t ring_bwd_ws(const usp::AttnGeom& g) {
  return usp::kStatusBytes + 2 * sizeof(float) * static_cast<size_t>(g.B) * g.Hq_l * padded(g);
}

// TMA maps of one rank's buffers [B][L][H][D] (bf16).
int local_tmap(CUtensorMap* m, const void* p, const usp::AttnGeom& g, int H) {
  const unsigned long long row = 2ull * H * g.D;
  return usp::make_tmap_strided(m, p, g.D, H, g.L, g.B, row, row * g.L);
}

int check_rank(const usp::AttnGeom& g, int i, int u, int t) {
  if (i < 0 || i >= g.P_r || u < 0 || u >= g.P_u || t < 0 || t >= g.P_r)
    return record_error(USP_ERR_INVALID_ARG, "rank (i=%d, u=%d) or step t=%d outside the %dx%d mesh", i, u, t, g.P_u,
                        g.P_r);
  return USP_OK;
}

}  // namespace

extern "C" {

int usp_ulysses_pack(int map, const usp_permute_job* jobs, int n_jobs, int B, int T, int G, void* stream) {
  if (map < USP_MAP_PACK_HEADS || map > USP_MAP_UNPACK_HEADS) return record_error(USP_ERR_INVALID_ARG, "bad map %d", map);
  if (!jobs || n_jobs <= 0 || n_jobs > usp::kMaxLayoutJobs)
    return record_error(USP_ERR_INVALID_ARG, "n_jobs must be 1..%d with a job array", usp::kMaxLayoutJobs);
  if (B <= 0 || T <= 0 || G <= 0) return record_error(USP_ERR_INVALID_ARG, "sizes must be positive");
  usp::LayoutArgs a[usp::kMaxLayoutJobs];
  for (int x = 0; x < n_jobs; ++x) {
    const usp_permute_job& j = jobs[x];
    const int es = elem_size(j.dtype);
    if (!j.src || !j.dst) return record_error(USP_ERR_INVALID_ARG, "job %d: null pointer", x);
    if (!aligned16(j.src) || !aligned16(j.dst))
      return record_error(USP_ERR_INVALID_ARG, "job %d: pointers must be 16-byte aligned", x);
    if (es == 0) return record_error(USP_ERR_INVALID_ARG, "job %d: dtype must be USP_BF16 or USP_F32", x);
    if (j.H <= 0 || j.D <= 0) return record_error(USP_ERR_INVALID_ARG, "job %d: sizes must be positive", x);
    if (j.H % G != 0) return record_error(USP_ERR_UNSUPPORTED, "job %d: H (%d) must be a multiple of G (%d)", x, j.H, G);
    if ((static_cast<long long>(j.D) * es) % 4 != 0)
      return record_error(USP_ERR_UNSUPPORTED, "job %d: D * element size must be a multiple of 4", x);
    if (static_cast<long long>(B) * T * G >= (1LL << 31)) return record_error(USP_ERR_UNSUPPORTED, "too many rows");
    a[x] = usp::LayoutArgs{};
    a[x].src = static_cast<const uint8_t*>(j.src);
    a[x].dst = static_cast<uint8_t*>(j.dst);
    a[x].map = map;  // the USP_MAP_* codes of these maps are the kernel's
    a[x].B = B; a[x].S = T; a[x].H = j.H; a[x].P_u = G; a[x].P_r = 1;
    a[x].row_bytes = static_cast<uint32_t>(j.D * es);
  }
  const cudaError_t e = usp::launch_layout_batch(a, n_jobs, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? USP_OK : record_error(USP_ERR_CUDA, "layout kernel launch: %s", cudaGetErrorString(e));
}

size_t usp_ring_workspace_size(int B, int S, int Hq, int Hkv, int D, int causal, int P_u, int P_r, int bwd) {
  usp::AttnGeom g{};
  if (usp::validate_geom(B, S, Hq, Hkv, D, causal, P_u, P_r, &g) != USP_OK) return 0;
  return bwd ? ring_bwd_ws(g) : static_cast<size_t>(usp::kStatusBytes);
}

}  // extern "C"

namespace {

int ring_fwd(const void* q, const void* k, const void* v, float* o_part, float* lse_part, int B, int S, int Hq,
             int Hkv, int D, int causal, int P_u, int P_r, int i, int u, int t, void* workspace, size_t ws_bytes,
             void* stream, bool fold) {
  usp::AttnGeom g{};
  int rc = usp::validate_geom(B, S, Hq, Hkv, D, causal, P_u, P_r, &g);
  if (rc != USP_OK) return rc;
  if ((rc = check_rank(g, i, u, t)) != USP_OK) return rc;
  if (!q || !k || !v || !o_part || !lse_part) return record_error(USP_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o_part) || !aligned16(lse_part))
    return record_error(USP_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  if (!workspace || ws_bytes < static_cast<size_t>(usp::kStatusBytes) || !aligned16(workspace))
    return record_error(USP_ERR_WORKSPACE, "workspace needs %d bytes (got %zu)", usp::kStatusBytes, ws_bytes);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  usp::FwdLaunch L{};
  L.g = g;
  if ((rc = local_tmap(&L.tm_q, q, g, g.Hq_l)) != USP_OK) return rc;
  if ((rc = local_tmap(&L.tm_k, k, g, g.Hkv_l)) != USP_OK) return rc;
  if ((rc = local_tmap(&L.tm_v, v, g, g.Hkv_l)) != USP_OK) return rc;
  L.status = static_cast<int*>(workspace);
  L.wait_ns = usp::current_wait_ns();
  L.step = t;
  L.o_part = o_part;
  L.lse_part = lse_part;
  L.local = 1;
  L.loc_i = i;
  L.loc_u = u;
  L.fold = fold ? 1 : 0;
  cudaError_t e = cudaMemsetAsync(workspace, 0, sizeof(int), st);
  if (e == cudaSuccess) e = usp::launch_attn_fwd(L, st);
  return e == cudaSuccess ? USP_OK : record_error(USP_ERR_CUDA, "ring step launch: %s", cudaGetErrorString(e));
}

}  // namespace

extern "C" {

int usp_ring_fwd_step(const void* q, const void* k, const void* v, float* o_part, float* lse_part, int B, int S,
                      int Hq, int Hkv, int D, int causal, int P_u, int P_r, int i, int u, int t, void* workspace,
                      size_t ws_bytes, void* stream) {
  return ring_fwd(q, k, v, o_part, lse_part, B, S, Hq, Hkv, D, causal, P_u, P_r, i, u, t, workspace, ws_bytes,
                  stream, false);
}

int usp_ring_fwd_accumulate(const void* q, const void* k, const void* v, float* o_run, float* lse_run, int B, int S,
                            int Hq, int Hkv, int D, int causal, int P_u, int P_r, int i, int u, int t,
                            void* workspace, size_t ws_bytes, void* stream) {
  return ring_fwd(q, k, v, o_run, lse_run, B, S, Hq, Hkv, D, causal, P_u, P_r, i, u, t, workspace, ws_bytes, stream,
                  t > 0);
}

int usp_ring_bwd_prepare(const void* out, const float* lse, const void* dO, int B, int S, int Hq, int Hkv, int D,
                         int causal, int P_u, int P_r, void* workspace, size_t ws_bytes, void* stream) {
  usp::AttnGeom g{};
  int rc = usp::validate_geom(B, S, Hq, Hkv, D, causal, P_u, P_r, &g);
  if (rc != USP_OK) return rc;
  if (!out || !lse || !dO) return record_error(USP_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(out) || !aligned16(lse) || !aligned16(dO))
    return record_error(USP_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  const size_t need = ring_bwd_ws(g);
  if (!workspace || ws_bytes < need || !aligned16(workspace))
    return record_error(USP_ERR_WORKSPACE, "workspace needs %zu bytes (got %zu)", need, ws_bytes);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int Lp = padded(g);
  float* lse2 = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + usp::kStatusBytes);
  float* delta = lse2 + static_cast<size_t>(B) * g.Hq_l * Lp;
  cudaError_t e = cudaMemsetAsync(workspace, 0, sizeof(int), st);
  if (e == cudaSuccess) e = usp::launch_bwd_prep_rows(out, dO, lse, delta, lse2, B, g.L, g.Hq_l, D, Lp, st);
  return e == cudaSuccess ? USP_OK : record_error(USP_ERR_CUDA, "preprocess launch: %s", cudaGetErrorString(e));
}

int usp_ring_bwd_step(const void* q, const void* k, const void* v, const void* dO, float* dq_acc, void* dq_out,
                      float* dk_acc, float* dv_acc, int B, int S, int Hq, int Hkv, int D, int causal, int P_u, int P_r,
                      int i, int u, int t, void* workspace, size_t ws_bytes, void* stream) {
  usp::AttnGeom g{};
  int rc = usp::validate_geom(B, S, Hq, Hkv, D, causal, P_u, P_r, &g);
  if (rc != USP_OK) return rc;
  if ((rc = check_rank(g, i, u, t)) != USP_OK) return rc;
  if (!q || !k || !v || !dO || !dq_acc || !dk_acc || !dv_acc) return record_error(USP_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dO) || !aligned16(dq_acc) ||
      !aligned16(dk_acc) || !aligned16(dv_acc) || (dq_out && !aligned16(dq_out)))
    return record_error(USP_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  const size_t need = ring_bwd_ws(g);
  if (!workspace || ws_bytes < need || !aligned16(workspace))
    return record_error(USP_ERR_WORKSPACE, "workspace needs %zu bytes (got %zu)", need, ws_bytes);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  usp::BwdLaunch L{};
  L.g = g;
  if ((rc = local_tmap(&L.tm_q, q, g, g.Hq_l)) != USP_OK) return rc;
  if ((rc = local_tmap(&L.tm_k, k, g, g.Hkv_l)) != USP_OK) return rc;
  if ((rc = local_tmap(&L.tm_v, v, g, g.Hkv_l)) != USP_OK) return rc;
  if ((rc = local_tmap(&L.tm_do, dO, g, g.Hq_l)) != USP_OK) return rc;
  const int Lp = padded(g);
  L.lse2 = reinterpret_cast<const float*>(static_cast<const uint8_t*>(workspace) + usp::kStatusBytes);
  L.delta = L.lse2 + static_cast<size_t>(B) * g.Hq_l * Lp;
  L.Lp = Lp;
  L.status = static_cast<int*>(workspace);
  L.wait_ns = usp::current_wait_ns();
  L.local = 1;
  L.loc_i = i;
  L.loc_u = u;
  L.loc_t = t;
  L.loc_j = (i - t + P_r) % P_r;
  L.dk = dk_acc;
  L.dv = dv_acc;
  L.dq = dq_out;
  L.dq_acc = dq_acc;
  cudaError_t e = usp::launch_attn_bwd(L, st);
  if (e == cudaSuccess) e = usp::launch_attn_bwd_dq(L, st);
  return e == cudaSuccess ? USP_OK : record_error(USP_ERR_CUDA, "ring backward step launch: %s", cudaGetErrorString(e));
}

}  // extern "C"
