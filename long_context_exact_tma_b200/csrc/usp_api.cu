// usp_api.cu -- the extern "C" entry points of libusp.so (declared in include/usp.h):
// argument validation, workspace accounting, TMA tensor maps and kernel launches.
#include <cudaTypedefs.h>
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "../../include/usp.h"
#include "usp_internal.h"

using namespace usp;

namespace {

thread_local char g_err[512] = "";
thread_local unsigned long long g_wait_ns = 2000000000ull;

int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof g_err, fmt, ap);
  va_end(ap);
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(USP_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int elem_size(int dtype) { return dtype == USP_BF16 ? 2 : dtype == USP_F32 ? 4 : 0; }

// Shapes of the layout calls: B*S*H*D elements, S % 2P == 0, H % P_u == 0.
int check_layout(const void* src, const void* dst, int B, int S, int H, int D, int dtype, int P_u, int P_r) {
  if (!src || !dst) return fail(USP_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(src) || !aligned16(dst)) return fail(USP_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  if (B <= 0 || S <= 0 || H <= 0 || D <= 0 || P_u <= 0 || P_r <= 0)
    return fail(USP_ERR_INVALID_ARG, "sizes must be positive");
  const int es = elem_size(dtype);
  if (es == 0) return fail(USP_ERR_INVALID_ARG, "dtype must be USP_BF16 or USP_F32");
  if ((static_cast<long long>(D) * es) % 4 != 0) return fail(USP_ERR_UNSUPPORTED, "D * element size must be a multiple of 4");
  const long long P = static_cast<long long>(P_u) * P_r;
  if (S % (2 * P) != 0) return fail(USP_ERR_UNSUPPORTED, "S (%d) must be a multiple of 2*P (%lld)", S, 2 * P);
  if (H % P_u != 0) return fail(USP_ERR_UNSUPPORTED, "H (%d) must be a multiple of P_u (%d)", H, P_u);
  if (static_cast<long long>(B) * S * P_u >= (1LL << 31)) return fail(USP_ERR_UNSUPPORTED, "too many rows");
  if (static_cast<long long>(H) * D * es >= (1LL << 31)) return fail(USP_ERR_UNSUPPORTED, "token row too large");
  return USP_OK;
}

int run_layout(int map, const void* src, void* dst, int B, int S, int H, int D, int dtype, int P_u, int P_r,
               void* stream) {
  int rc = check_layout(src, dst, B, S, H, D, dtype, P_u, P_r);
  if (rc != USP_OK) return rc;
  LayoutArgs a{};
  a.src = static_cast<const uint8_t*>(src);
  a.dst = static_cast<uint8_t*>(dst);
  a.map = map;
  a.B = B; a.S = S; a.H = H; a.P_u = P_u; a.P_r = P_r;
  a.row_bytes = static_cast<uint32_t>(D * elem_size(dtype));
  cudaError_t e = launch_layout(a, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? USP_OK : cuda_fail(e, "layout kernel launch");
}

int run_layout_batch(int map, const usp_permute_job* jobs, int n, int B, int S, int P_u, int P_r, void* stream) {
  if (map < kZigzagShard || map > kHead2Seq) return fail(USP_ERR_INVALID_ARG, "bad map %d", map);
  if (!jobs || n <= 0 || n > kMaxLayoutJobs)
    return fail(USP_ERR_INVALID_ARG, "n_jobs must be 1..%d with a job array", kMaxLayoutJobs);
  LayoutArgs a[kMaxLayoutJobs];
  for (int x = 0; x < n; ++x) {
    const usp_permute_job& j = jobs[x];
    const int rc = check_layout(j.src, j.dst, B, S, j.H, j.D, j.dtype, P_u, P_r);
    if (rc != USP_OK) {
      char why[sizeof g_err];
      snprintf(why, sizeof why, "%s", g_err);
      return fail(rc, "job %d: %s", x, why);
    }
    a[x] = LayoutArgs{};
    a[x].src = static_cast<const uint8_t*>(j.src);
    a[x].dst = static_cast<uint8_t*>(j.dst);
    a[x].map = map;
    a[x].B = B; a[x].S = S; a[x].H = j.H; a[x].P_u = P_u; a[x].P_r = P_r;
    a[x].row_bytes = static_cast<uint32_t>(j.D * elem_size(j.dtype));
  }
  cudaError_t e = launch_layout_batch(a, n, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? USP_OK : cuda_fail(e, "layout kernel launch");
}

int check_geom(int B, int S, int Hq, int Hkv, int D, int causal, int P_u, int P_r, AttnGeom* g) {
  if (B <= 0 || S <= 0 || Hq <= 0 || Hkv <= 0 || P_u <= 0 || P_r <= 0)
    return fail(USP_ERR_INVALID_ARG, "sizes must be positive");
  if (causal != 0 && causal != 1) return fail(USP_ERR_INVALID_ARG, "causal must be 0 or 1");
  if (D != 64 && D != 128) return fail(USP_ERR_UNSUPPORTED, "D must be 64 or 128 (got %d)", D);
  if (Hq % Hkv != 0) return fail(USP_ERR_UNSUPPORTED, "Hq %% Hkv != 0");
  if (Hq % P_u != 0 || Hkv % P_u != 0) return fail(USP_ERR_UNSUPPORTED, "Hq and Hkv must be multiples of P_u");
  const long long P = static_cast<long long>(P_u) * P_r;
  if (S % (2 * P) != 0) return fail(USP_ERR_UNSUPPORTED, "S (%d) must be a multiple of 2*P (%lld)", S, 2 * P);
  if (static_cast<long long>(B) * S * Hq >= (1LL << 31)) return fail(USP_ERR_UNSUPPORTED, "too many rows");
  g->B = B; g->S = S; g->Hq = Hq; g->Hkv = Hkv; g->D = D; g->causal = causal; g->P_u = P_u; g->P_r = P_r;
  g->P = static_cast<int>(P);
  g->c = S / (2 * g->P);
  g->L = S / P_r;
  g->Hq_l = Hq / P_u;
  g->Hkv_l = Hkv / P_u;
  g->G = Hq / Hkv;
  g->n_ranks = P_r * P_u;
  return USP_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q{};
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Head-sharded bf16 tensor [n_rb][L][H_l][D] viewed as 4-D {D, H_l, L, n_rb};
// box = 64 elements (128 B, one swizzle panel) x 1 head x 128 rows x 1.
int make_tmap(CUtensorMap* m, const void* base, int D, int H_l, int L, int n_rb) {
  auto fn = encode_fn();
  if (!fn) return fail(USP_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H_l), static_cast<cuuint64_t>(L),
                        static_cast<cuuint64_t>(n_rb)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(H_l) * D * 2,
                           static_cast<cuuint64_t>(L) * H_l * D * 2};
  cuuint32_t box[4] = {64, 1, 128, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(USP_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return USP_OK;
}

}  // namespace

namespace usp {
// Tensor map of a bf16 tensor viewed as 4-D {D, H, rows, n4}: head rows of D
// elements 2*D bytes apart, `rows` rows row_stride bytes apart and n4 blocks
// stride4 bytes apart; box 64 x 1 x 128 x 1, 128-byte swizzle.
int make_tmap_strided(CUtensorMap* m, const void* base, int D, int H, long long rows, long long n4,
                      unsigned long long row_stride, unsigned long long stride4) {
  return make_tmap_strided_h(m, base, D, H, rows, n4, static_cast<unsigned long long>(D) * 2, row_stride, stride4);
}
int make_tmap_strided_h(CUtensorMap* m, const void* base, int D, int H, long long rows, long long n4,
                        unsigned long long head_stride, unsigned long long row_stride, unsigned long long stride4) {
  auto fn = encode_fn();
  if (!fn) return record_error(USP_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(n4)};
  cuuint64_t strides[3] = {head_stride, row_stride, stride4};
  cuuint32_t box[4] = {64, 1, 128, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return record_error(USP_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return USP_OK;
}
unsigned long long current_wait_ns() { return g_wait_ns; }

namespace {
struct SidePool {
  int dev = -1;
  cudaStream_t s[kSideStreams];
  cudaEvent_t fork;
  cudaEvent_t join[kSideStreams];
};
thread_local SidePool t_side;

cudaError_t side_pool(SidePool** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  SidePool& p = t_side;
  if (p.dev != dev) {  // first use on this device by this thread
    for (int i = 0; i < kSideStreams && e == cudaSuccess; ++i) {
      e = cudaStreamCreateWithFlags(&p.s[i], cudaStreamNonBlocking);
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p.join[i], cudaEventDisableTiming);
    }
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p.fork, cudaEventDisableTiming);
    if (e != cudaSuccess) return e;
    p.dev = dev;
  }
  *out = &p;
  return cudaSuccess;
}
}  // namespace

cudaError_t side_fork(cudaStream_t main, int n, cudaStream_t* out) {
  SidePool* p = nullptr;
  cudaError_t e = side_pool(&p);
  if (e == cudaSuccess) e = cudaEventRecord(p->fork, main);
  for (int i = 0; i < n && i < kSideStreams && e == cudaSuccess; ++i) {
    e = cudaStreamWaitEvent(p->s[i], p->fork, 0);
    out[i] = p->s[i];
  }
  return e;
}

cudaError_t side_join(cudaStream_t main, int n) {
  SidePool* p = nullptr;
  cudaError_t e = side_pool(&p);
  for (int i = 0; i < n && i < kSideStreams && e == cudaSuccess; ++i) {
    e = cudaEventRecord(p->join[i], p->s[i]);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(main, p->join[i], 0);
  }
  return e;
}
}  // namespace usp

namespace {
int check_geom(int B, int S, int Hq, int Hkv, int D, int causal, int P_u, int P_r, AttnGeom* g);
}  // namespace

namespace usp {
int validate_geom(int B, int S, int Hq, int Hkv, int D, int causal, int P_u, int P_r, AttnGeom* g) {
  return check_geom(B, S, Hq, Hkv, D, causal, P_u, P_r, g);
}
}  // namespace usp

namespace {

size_t rows_of(const AttnGeom& g) { return static_cast<size_t>(g.B) * g.S * g.Hq; }

// Stepwise mode streams the merge: two fp32 partials, the running merge of the
// steps done so far (slot 0) and the current step's partial (slot 1).
size_t fwd_ws(const AttnGeom& g, int mode) {
  if (mode == USP_MODE_FUSED) return kStatusBytes;
  return kStatusBytes + 2 * rows_of(g) * (4 * static_cast<size_t>(g.D) + 4);
}
int padded_L(const AttnGeom& g) { return (g.L + 127) / 128 * 128; }
// [status][-LSE*log2e per head: n_rb*Hq_l*Lp][-Delta per head: same]
size_t bwd_ws(const AttnGeom& g) {
  const size_t per_head = static_cast<size_t>(g.n_ranks) * g.B * g.Hq_l * padded_L(g);
  return kStatusBytes + 2 * per_head * 4;
}

}  // namespace

namespace usp {
namespace {
std::atomic<unsigned long long> g_launches{0};
}  // namespace
void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

// Records `msg` as this thread's last error and returns `code` (for entry points in other files).
int record_error(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof g_err, fmt, ap);
  va_end(ap);
  return code;
}
}  // namespace usp

extern "C" {

int usp_version(void) { return 100; }

const char* usp_last_error(void) { return g_err; }

unsigned long long usp_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

void usp_set_wait_limit_ns(unsigned long long ns) { g_wait_ns = ns; }

int usp_zigzag_shard(const void* src, void* dst, int B, int S, int H, int D, int dtype, int P_u, int P_r,
                     void* stream) {
  return run_layout(kZigzagShard, src, dst, B, S, H, D, dtype, P_u, P_r, stream);
}
int usp_zigzag_unshard(const void* src, void* dst, int B, int S, int H, int D, int dtype, int P_u, int P_r,
                       void* stream) {
  return run_layout(kZigzagUnshard, src, dst, B, S, H, D, dtype, P_u, P_r, stream);
}
int usp_seq2head_permute(const void* src, void* dst, int B, int S, int H, int D, int dtype, int P_u, int P_r,
                         void* stream) {
  return run_layout(kSeq2Head, src, dst, B, S, H, D, dtype, P_u, P_r, stream);
}
int usp_head2seq_permute(const void* src, void* dst, int B, int S, int H, int D, int dtype, int P_u, int P_r,
                         void* stream) {
  return run_layout(kHead2Seq, src, dst, B, S, H, D, dtype, P_u, P_r, stream);
}

int usp_permute_batch(int map, const usp_permute_job* jobs, int n_jobs, int B, int S, int P_u, int P_r,
                      void* stream) {
  static_assert(USP_MAX_PERMUTE_JOBS == kMaxLayoutJobs, "job limit");
  static_assert(USP_MAP_SEQ2HEAD == kSeq2Head && USP_MAP_HEAD2SEQ == kHead2Seq && USP_MAP_ZIGZAG_SHARD == kZigzagShard &&
                    USP_MAP_ZIGZAG_UNSHARD == kZigzagUnshard,
                "map codes");
  return run_layout_batch(map, jobs, n_jobs, B, S, P_u, P_r, stream);
}

size_t usp_attn_workspace_size(int B, int S, int Hq, int Hkv, int D, int causal, int P_u, int P_r, int mode,
                               int bwd) {
  AttnGeom g{};
  if (check_geom(B, S, Hq, Hkv, D, causal, P_u, P_r, &g) != USP_OK) return 0;
  if (bwd) return bwd_ws(g);
  if (mode != USP_MODE_FUSED && mode != USP_MODE_STEPWISE) return 0;
  return fwd_ws(g, mode);
}

}  // extern "C"

namespace {

// The masks of usp_attn_*_masked as kernel arguments; validates them against
// the geometry (masks need chunks that are whole tiles).
int mask_args(const usp_attn_mask* m, const AttnGeom& g, MaskArgs* out) {
  *out = MaskArgs{};
  if (!m || (!m->block_mask && !m->cu_seqlens)) return USP_OK;
  if (g.c % 128 != 0)
    return fail(USP_ERR_UNSUPPORTED, "masks need zigzag chunks of a multiple of 128 tokens (S/(2 P) = %d)", g.c);
  if (m->cu_seqlens && m->n_docs < 1) return fail(USP_ERR_INVALID_ARG, "n_docs must be >= 1 with cu_seqlens");
  out->bm = m->block_mask;
  out->cu = m->cu_seqlens;
  out->n_docs = m->cu_seqlens ? m->n_docs : 0;
  out->nb = g.S / 128;
  out->Hq = g.Hq;
  return USP_OK;
}

int attn_fwd_impl(const void* q, const void* k, const void* v, void* out, float* lse, int B, int S, int Hq, int Hkv,
                  int D, int causal, int P_u, int P_r, int mode, const usp_attn_mask* mask, void* workspace,
                  size_t ws_bytes, void* stream) {
  AttnGeom g{};
  int rc = check_geom(B, S, Hq, Hkv, D, causal, P_u, P_r, &g);
  if (rc != USP_OK) return rc;
  MaskArgs mk{};
  if ((rc = mask_args(mask, g, &mk)) != USP_OK) return rc;
  if (mode != USP_MODE_FUSED && mode != USP_MODE_STEPWISE) return fail(USP_ERR_INVALID_ARG, "bad mode %d", mode);
  if (!q || !k || !v || !out || !lse) return fail(USP_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse))
    return fail(USP_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  const size_t need = fwd_ws(g, mode);
  if (!workspace || ws_bytes < need || !aligned16(workspace))
    return fail(USP_ERR_WORKSPACE, "workspace needs %zu bytes (got %zu)", need, ws_bytes);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  FwdLaunch L{};
  L.g = g;
  if ((rc = make_tmap(&L.tm_q, q, D, g.Hq_l, g.L, g.n_ranks * B)) != USP_OK) return rc;
  if ((rc = make_tmap(&L.tm_k, k, D, g.Hkv_l, g.L, g.n_ranks * B)) != USP_OK) return rc;
  if ((rc = make_tmap(&L.tm_v, v, D, g.Hkv_l, g.L, g.n_ranks * B)) != USP_OK) return rc;
  L.status = static_cast<int*>(workspace);
  L.wait_ns = g_wait_ns;
  L.mask = mk;
  cudaError_t e = cudaMemsetAsync(workspace, 0, sizeof(int), st);
  if (e != cudaSuccess) return cuda_fail(e, "status reset");
  if (mode == USP_MODE_FUSED) {
    L.out = out;
    L.lse = lse;
    L.step = -1;
    e = launch_attn_fwd(L, st);
    return e == cudaSuccess ? USP_OK : cuda_fail(e, "attention forward launch");
  }
  // The ring step for step: step t's partial goes to slot 1 (step 0's to slot 0)
  // and is folded into the running result in slot 0 by the log-sum-exp merge,
  // 2 partials in and 1 out; the last step's merge writes O (bf16) and LSE.
  const size_t rows = rows_of(g);
  float* o_parts = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kStatusBytes);
  float* lse_parts = o_parts + 2 * rows * D;
  for (int t = 0; t < P_r; ++t) {
    const int slot = t == 0 ? 0 : 1;
    L.step = t;
    L.o_part = o_parts + static_cast<size_t>(slot) * rows * D;
    L.lse_part = lse_parts + static_cast<size_t>(slot) * rows;
    e = launch_attn_fwd(L, st);
    if (e != cudaSuccess) return cuda_fail(e, "attention forward (step) launch");
    const bool last = t == P_r - 1;
    if (t == 0 && !last) continue;
    e = last ? launch_lse_merge(o_parts, lse_parts, t == 0 ? 1 : 2, static_cast<long long>(rows), D, out, 0, lse,
                                st)
             : launch_lse_merge(o_parts, lse_parts, 2, static_cast<long long>(rows), D, o_parts, 1, lse_parts, st);
    if (e != cudaSuccess) return cuda_fail(e, "merge launch");
  }
  return USP_OK;
}

}  // namespace

extern "C" {

int usp_attn_fwd(const void* q, const void* k, const void* v, void* out, float* lse, int B, int S, int Hq,
                 int Hkv, int D, int causal, int P_u, int P_r, int mode, void* workspace, size_t ws_bytes,
                 void* stream) {
  return attn_fwd_impl(q, k, v, out, lse, B, S, Hq, Hkv, D, causal, P_u, P_r, mode, nullptr, workspace, ws_bytes,
                       stream);
}

int usp_attn_fwd_masked(const void* q, const void* k, const void* v, void* out, float* lse, int B, int S, int Hq,
                        int Hkv, int D, int causal, int P_u, int P_r, const usp_attn_mask* mask, void* workspace,
                        size_t ws_bytes, void* stream) {
  return attn_fwd_impl(q, k, v, out, lse, B, S, Hq, Hkv, D, causal, P_u, P_r, USP_MODE_FUSED, mask, workspace,
                       ws_bytes, stream);
}

int usp_attn_bwd_prepare(const void* out, const float* lse, const void* dO, int B, int S, int Hq, int Hkv, int D,
                         int causal, int P_u, int P_r, void* workspace, size_t ws_bytes, void* stream) {
  AttnGeom g{};
  int rc = check_geom(B, S, Hq, Hkv, D, causal, P_u, P_r, &g);
  if (rc != USP_OK) return rc;
  if (!out || !lse || !dO) return fail(USP_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(out) || !aligned16(lse) || !aligned16(dO))
    return fail(USP_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  const size_t need = bwd_ws(g);
  if (!workspace || ws_bytes < need || !aligned16(workspace))
    return fail(USP_ERR_WORKSPACE, "workspace needs %zu bytes (got %zu)", need, ws_bytes);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int Lp = padded_L(g);
  const size_t per_head = static_cast<size_t>(g.n_ranks) * B * g.Hq_l * Lp;
  float* lse2 = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kStatusBytes);
  float* delta = lse2 + per_head;
  cudaError_t e = cudaMemsetAsync(workspace, 0, sizeof(int), st);
  if (e != cudaSuccess) return cuda_fail(e, "workspace reset");
  e = launch_bwd_prep_rows(out, dO, lse, delta, lse2, g.n_ranks * B, g.L, g.Hq_l, D, Lp, st);
  return e == cudaSuccess ? USP_OK : cuda_fail(e, "preprocess launch");
}

}  // extern "C"

namespace {
// Validation and TMA maps shared by the two backward kernels (workspace prepared
// by usp_attn_bwd_prepare).
int bwd_launch_setup(const void* q, const void* k, const void* v, const void* dO, int B, int S, int Hq, int Hkv,
                     int D, int causal, int P_u, int P_r, const usp_attn_mask* mask, void* workspace,
                     size_t ws_bytes, BwdLaunch* L) {
  AttnGeom g{};
  int rc = check_geom(B, S, Hq, Hkv, D, causal, P_u, P_r, &g);
  if (rc != USP_OK) return rc;
  if ((rc = mask_args(mask, g, &L->mask)) != USP_OK) return rc;
  if (!q || !k || !v || !dO) return fail(USP_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dO))
    return fail(USP_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  const size_t need = bwd_ws(g);
  if (!workspace || ws_bytes < need || !aligned16(workspace))
    return fail(USP_ERR_WORKSPACE, "workspace needs %zu bytes (got %zu)", need, ws_bytes);
  const int Lp = padded_L(g);
  const size_t per_head = static_cast<size_t>(g.n_ranks) * B * g.Hq_l * Lp;
  L->g = g;
  if ((rc = make_tmap(&L->tm_q, q, D, g.Hq_l, g.L, g.n_ranks * B)) != USP_OK) return rc;
  if ((rc = make_tmap(&L->tm_k, k, D, g.Hkv_l, g.L, g.n_ranks * B)) != USP_OK) return rc;
  if ((rc = make_tmap(&L->tm_v, v, D, g.Hkv_l, g.L, g.n_ranks * B)) != USP_OK) return rc;
  if ((rc = make_tmap(&L->tm_do, dO, D, g.Hq_l, g.L, g.n_ranks * B)) != USP_OK) return rc;
  L->lse2 = reinterpret_cast<const float*>(static_cast<const uint8_t*>(workspace) + kStatusBytes);
  L->delta = L->lse2 + per_head;
  L->Lp = Lp;
  L->status = static_cast<int*>(workspace);
  L->wait_ns = g_wait_ns;
  return USP_OK;
}

// dK, dV in fp32 (bf16 = 0) or, rounded once from the fp32 sums, in bf16 (bf16 = 1)
int bwd_dkdv_impl(const void* q, const void* k, const void* v, const void* dO, void* dK, void* dV, int bf16, int B,
                  int S, int Hq, int Hkv, int D, int causal, int P_u, int P_r, const usp_attn_mask* mask,
                  void* workspace, size_t ws_bytes, void* stream) {
  if (!dK || !dV) return fail(USP_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(dK) || !aligned16(dV)) return fail(USP_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  BwdLaunch L{};
  const int rc = bwd_launch_setup(q, k, v, dO, B, S, Hq, Hkv, D, causal, P_u, P_r, mask, workspace, ws_bytes, &L);
  if (rc != USP_OK) return rc;
  if (bf16) {
    L.dk_bf16 = dK;
    L.dv_bf16 = dV;
  } else {
    L.dk = static_cast<float*>(dK);
    L.dv = static_cast<float*>(dV);
  }
  const cudaError_t e = launch_attn_bwd(L, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? USP_OK : cuda_fail(e, "attention backward (dK, dV) launch");
}

int bwd_dq_impl(const void* q, const void* k, const void* v, const void* dO, void* dQ, int B, int S, int Hq, int Hkv,
                int D, int causal, int P_u, int P_r, const usp_attn_mask* mask, void* workspace, size_t ws_bytes,
                void* stream) {
  if (!dQ) return fail(USP_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(dQ)) return fail(USP_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  BwdLaunch L{};
  const int rc = bwd_launch_setup(q, k, v, dO, B, S, Hq, Hkv, D, causal, P_u, P_r, mask, workspace, ws_bytes, &L);
  if (rc != USP_OK) return rc;
  L.dq = dQ;
  const cudaError_t e = launch_attn_bwd_dq(L, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? USP_OK : cuda_fail(e, "attention backward (dQ) launch");
}

int attn_bwd_impl(const void* q, const void* k, const void* v, const void* out, const float* lse, const void* dO,
                  void* dQ, float* dK, float* dV, int B, int S, int Hq, int Hkv, int D, int causal, int P_u, int P_r,
                  const usp_attn_mask* mask, void* workspace, size_t ws_bytes, void* stream) {
  AttnGeom g{};
  int rc = check_geom(B, S, Hq, Hkv, D, causal, P_u, P_r, &g);
  if (rc != USP_OK) return rc;
  MaskArgs mk{};
  if ((rc = mask_args(mask, g, &mk)) != USP_OK) return rc;
  if (!q || !k || !v || !out || !lse || !dO || !dQ || !dK || !dV) return fail(USP_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse) || !aligned16(dO) ||
      !aligned16(dQ) || !aligned16(dK) || !aligned16(dV))
    return fail(USP_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  if ((rc = usp_attn_bwd_prepare(out, lse, dO, B, S, Hq, Hkv, D, causal, P_u, P_r, workspace, ws_bytes, stream)) !=
      USP_OK)
    return rc;
  if ((rc = bwd_dkdv_impl(q, k, v, dO, dK, dV, 0, B, S, Hq, Hkv, D, causal, P_u, P_r, mask, workspace, ws_bytes,
                          stream)) != USP_OK)
    return rc;
  return bwd_dq_impl(q, k, v, dO, dQ, B, S, Hq, Hkv, D, causal, P_u, P_r, mask, workspace, ws_bytes, stream);
}
}  // namespace

extern "C" {

int usp_attn_bwd_dkdv(const void* q, const void* k, const void* v, const void* dO, float* dK, float* dV, int B,
                      int S, int Hq, int Hkv, int D, int causal, int P_u, int P_r, void* workspace, size_t ws_bytes,
                      void* stream) {
  return bwd_dkdv_impl(q, k, v, dO, dK, dV, 0, B, S, Hq, Hkv, D, causal, P_u, P_r, nullptr, workspace, ws_bytes,
                       stream);
}

int usp_attn_bwd_dkdv_bf16(const void* q, const void* k, const void* v, const void* dO, void* dK, void* dV, int B,
                           int S, int Hq, int Hkv, int D, int causal, int P_u, int P_r, void* workspace,
                           size_t ws_bytes, void* stream) {
  return bwd_dkdv_impl(q, k, v, dO, dK, dV, 1, B, S, Hq, Hkv, D, causal, P_u, P_r, nullptr, workspace, ws_bytes,
                       stream);
}

int usp_attn_bwd_dq(const void* q, const void* k, const void* v, const void* dO, void* dQ, int B, int S, int Hq,
                    int Hkv, int D, int causal, int P_u, int P_r, void* workspace, size_t ws_bytes, void* stream) {
  return bwd_dq_impl(q, k, v, dO, dQ, B, S, Hq, Hkv, D, causal, P_u, P_r, nullptr, workspace, ws_bytes, stream);
}

int usp_attn_bwd(const void* q, const void* k, const void* v, const void* out, const float* lse, const void* dO,
                 void* dQ, float* dK, float* dV, int B, int S, int Hq, int Hkv, int D, int causal, int P_u,
                 int P_r, void* workspace, size_t ws_bytes, void* stream) {
  return attn_bwd_impl(q, k, v, out, lse, dO, dQ, dK, dV, B, S, Hq, Hkv, D, causal, P_u, P_r, nullptr, workspace,
                       ws_bytes, stream);
}

int usp_attn_bwd_masked(const void* q, const void* k, const void* v, const void* out, const float* lse,
                        const void* dO, void* dQ, float* dK, float* dV, int B, int S, int Hq, int Hkv, int D,
                        int causal, int P_u, int P_r, const usp_attn_mask* mask, void* workspace, size_t ws_bytes,
                        void* stream) {
  return attn_bwd_impl(q, k, v, out, lse, dO, dQ, dK, dV, B, S, Hq, Hkv, D, causal, P_u, P_r, mask, workspace,
                       ws_bytes, stream);
}

int usp_lse_merge(const float* o_parts, const float* lse_parts, int n_parts, long long rows, int D, void* out,
                  int out_dtype, float* lse_out, void* stream) {
  if (!o_parts || !lse_parts || !out || !lse_out) return fail(USP_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(o_parts) || !aligned16(out)) return fail(USP_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  if (n_parts <= 0 || rows < 0 || D <= 0) return fail(USP_ERR_INVALID_ARG, "sizes must be positive");
  if (D % 4 != 0 || D > 256) return fail(USP_ERR_UNSUPPORTED, "D must be a multiple of 4, at most 256");
  if (out_dtype != USP_BF16 && out_dtype != USP_F32) return fail(USP_ERR_INVALID_ARG, "bad out_dtype");
  cudaError_t e = launch_lse_merge(o_parts, lse_parts, n_parts, rows, D, out, out_dtype == USP_F32, lse_out,
                                   static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? USP_OK : cuda_fail(e, "merge launch");
}

int usp_bwd_preprocess(const void* out, const void* dO, float* delta, long long rows, int D, void* stream) {
  if (!out || !dO || !delta) return fail(USP_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(out) || !aligned16(dO)) return fail(USP_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  if (rows < 0 || D <= 0) return fail(USP_ERR_INVALID_ARG, "sizes must be positive");
  if (D % 4 != 0) return fail(USP_ERR_UNSUPPORTED, "D must be a multiple of 4");
  cudaError_t e = launch_bwd_preprocess(out, dO, delta, rows, D, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? USP_OK : cuda_fail(e, "preprocess launch");
}

int usp_workspace_status(void* workspace, int* site, void* stream) {
  if (!workspace) return fail(USP_ERR_INVALID_ARG, "null workspace");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int word = 0;
  cudaError_t e = cudaMemcpyAsync(&word, workspace, sizeof(int), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e == cudaSuccess) e = cudaMemsetAsync(workspace, 0, sizeof(int), st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "status read");
  if (site) *site = word;
  if (word != 0) return fail(USP_ERR_TIMEOUT, "a device wait timed out (site 0x%x)", word);
  return USP_OK;
}

int usp_selftest_wait_timeout(void* workspace, size_t ws_bytes, unsigned long long limit_ns, void* stream) {
  if (!workspace || ws_bytes < static_cast<size_t>(kStatusBytes))
    return fail(USP_ERR_WORKSPACE, "workspace needs %d bytes", kStatusBytes);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(workspace, 0, sizeof(int), st);
  if (e == cudaSuccess) e = launch_wait_selftest(static_cast<int*>(workspace), limit_ns, st);
  return e == cudaSuccess ? USP_OK : cuda_fail(e, "self-test launch");
}

}  // extern "C"
