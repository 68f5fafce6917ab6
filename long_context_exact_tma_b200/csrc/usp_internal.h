// usp_internal.h -- launch interfaces shared by the .cu files of libusp.so.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace usp {

constexpr int kStatusBytes = 256;  // workspace header: device status word + padding

// Sets the calling thread's usp_last_error() message; returns `code`.
int record_error(int code, const char* fmt, ...);

// Counts one kernel launch of this library (read by usp_launch_count).
void note_launch();

// The calling thread's bounded-wait limit (usp_set_wait_limit_ns).
unsigned long long current_wait_ns();

// Streams of the calling thread on the current device for launches that may
// run at the same time: side_fork makes n (<= kSideStreams) of them wait for
// the work issued so far on `main` and returns them; side_join makes `main`
// wait for everything issued on them since. Created on first use, kept for the
// thread's life (one set per thread, so concurrent callers never share an event).
constexpr int kSideStreams = 16;
cudaError_t side_fork(cudaStream_t main, int n, cudaStream_t* out);
cudaError_t side_join(cudaStream_t main, int n);

struct AttnGeom;
// The shape checks of the attention calls; fills g; usp_status (message recorded).
int validate_geom(int B, int S, int Hq, int Hkv, int D, int causal, int P_u, int P_r, AttnGeom* g);

// Tensor map of a bf16 tensor viewed as {D, H, rows, n4} with the given row and
// block strides in bytes (box 64 x 1 x 128 x 1, 128-byte swizzle); usp_status.
int make_tmap_strided(CUtensorMap* m, const void* base, int D, int H, long long rows, long long n4,
                      unsigned long long row_stride, unsigned long long stride4);
// The same with an explicit head stride in bytes (a multiple of 16).
int make_tmap_strided_h(CUtensorMap* m, const void* base, int D, int H, long long rows, long long n4,
                        unsigned long long head_stride, unsigned long long row_stride, unsigned long long stride4);

// Fills a running fp32 (O, LSE) with the empty result: O = 0, LSE = -inf.
cudaError_t launch_fill_running(float* o, float* lse, long long rows, int D, cudaStream_t stream);

// Layout maps of the gather kernel (see usp_layout.cu).
// The last four are the local halves of a real Ulysses all-to-all between G
// ranks holding T tokens each (run = the H/G heads of a group):
//   kPackHeads    [B][T][G][run] -> [G][B][T][run]  (send buffer of seq->head)
//   kUnpackTokens [G][B][T][run] -> [B][G][T][run]  (receive buffer of seq->head)
//   kPackTokens   [B][G][T][run] -> [G][B][T][run]  (send buffer of head->seq)
//   kUnpackHeads  [G][B][T][run] -> [B][T][G][run]  (receive buffer of head->seq)
// For these, LayoutArgs.S is T, P_u is G and P_r is 1.
enum LayoutMap {
  kZigzagShard = 0, kZigzagUnshard = 1, kSeq2Head = 2, kHead2Seq = 3,
  kPackHeads = 4, kUnpackTokens = 5, kPackTokens = 6, kUnpackHeads = 7
};

struct LayoutArgs {
  const uint8_t* src;
  uint8_t* dst;
  int map;
  uint32_t B, S, H, P_u, P_r;  // tokens, heads, mesh
  uint32_t row_bytes;          // bytes of one head row (D * element size)
};
cudaError_t launch_layout(const LayoutArgs& a, cudaStream_t stream);
// Up to kMaxLayoutJobs gathers in one launch (each with its own map, shape and
// element size).
constexpr int kMaxLayoutJobs = 4;
cudaError_t launch_layout_batch(const LayoutArgs* a, int n, cudaStream_t stream);

cudaError_t launch_lse_merge(const float* o_parts, const float* lse_parts, int n_parts, long long rows, int D,
                             void* out, int out_f32, float* lse_out, cudaStream_t stream);
cudaError_t launch_bwd_preprocess(const void* out, const void* dO, float* delta, long long rows, int D,
                                  cudaStream_t stream);
cudaError_t launch_wait_selftest(int* status, unsigned long long limit_ns, cudaStream_t stream);

// Block-sparse / document masks of the masked attention variants (see
// usp_attn_common.cuh); all null for plain causal or full attention.
struct MaskArgs {
  const uint8_t* bm;  // [B][Hq][nb][nb] block mask over 128-position blocks, or null
  const int* cu;      // [n_docs + 1] document boundaries, or null
  int nb, n_docs, Hq;
};

// Geometry of one attention problem in the head-sharded layout.
struct AttnGeom {
  int B, S, Hq, Hkv, D, causal, P_u, P_r;
  int P, c, L, Hq_l, Hkv_l, G;  // derived
  int n_ranks;                  // P_r * P_u head-sharded ranks
};

// The forward's sub-problem mode: one launch over n_prob independent one-rank
// problems of L rows each (plain order; the 4th TMA coordinate selects the
// problem), query heads h0 + j*h_step (j < n_heads). The result of row tau of
// problem p is folded into a running fp32 (O, LSE) at output row
// (p / n_seg) * S + (p % n_seg) * w + off + tau * r by the log-sum-exp merge.
// LongNet's dilated attention runs one such launch per (w, r) pair and head
// offset off, with tensor maps that step r rows from the offset.
// A query window makes a launch a cross-attention of some rows to the whole
// problem: Lq query rows whose kept indices (positions) start at q_off, against
// all L key rows (one rank's kept rows of a segment gathered from several
// ranks, LongNet's distributed layout). Query-side outputs (O, LSE, dQ, the row
// tables) use the mapping above with the output head out_h0 + h * out_hstep of
// the launch's head index h; the key-side outputs of the backward (dK, dV) use
// row (p / n_seg) * kS + (p % n_seg) * kw + koff + tau * kstep with kH heads a
// row. sub_defaults() makes a plain dilated launch: the window is all L rows,
// the output head is h, and keys map like queries.
struct FwdSub {
  int active;
  int n_prob, L, h0, h_step, n_heads;
  int n_seg, w, off, r, S, Hq;
  float* o_run;    // fp32 [B*S][Hq][D]
  float* lse_run;  // fp32 [B*S][Hq]
  int Lq, q_off;
  int out_h0, out_hstep;
  int kS, kw, koff, kstep, kH;
  // kv heads the dK/dV launch walks: kv0 + x * kv_step for x < n_kv (n_kv = 0: all)
  int kv0, kv_step, n_kv;
  // forward: the launch's rows hold nothing yet (a pair with r = 1 run first): write
  // the running (O, LSE) instead of folding into it, without reading it
  int first;
};
inline void sub_defaults(FwdSub& sb, int Hkv) {
  sb.Lq = sb.L;
  sb.q_off = 0;
  sb.out_h0 = 0;
  sb.out_hstep = 1;
  sb.kS = sb.S;
  sb.kw = sb.w;
  sb.koff = sb.off;
  sb.kstep = sb.r;
  sb.kH = Hkv;
  sb.kv0 = 0;
  sb.kv_step = 1;
  sb.n_kv = 0;
  sb.first = 0;
}

struct FwdLaunch {
  AttnGeom g;
  CUtensorMap tm_q, tm_k, tm_v;
  void* out;          // bf16 head-sharded (fused mode)
  float* lse;         // fp32 [ranks][B][L][Hq_l] (fused mode)
  float* o_part;      // fp32 partial O of one ring step (stepwise mode)
  float* lse_part;    // fp32 partial LSE of one ring step (stepwise mode)
  int step;           // ring step (stepwise) or -1 (fused)
  int* status;
  unsigned long long wait_ns;
  FwdSub sub;         // sub-problem mode when sub.active
  MaskArgs mask;      // masked variant when mask.bm or mask.cu is set
  int local;          // local mode: one rank (loc_i, loc_u) of a real mesh, its own buffers (B in dim 4)
  int loc_i, loc_u;
  int fold;           // stepwise / local: fold into o_part / lse_part (log-sum-exp merge) instead of writing
};
cudaError_t launch_attn_fwd(const FwdLaunch& a, cudaStream_t stream);

// Backward preprocess into the per-head layout the backward kernel streams:
// delta_t/lse2_t [n_ranks*B*Hq_l][Lp] (Lp = L rounded up to 128), holding -Delta
// and -LSE*log2(e); padding rows hold 0 and -inf.
cudaError_t launch_bwd_prep_rows(const void* out, const void* dO, const float* lse, float* delta_t, float* lse2_t,
                                 int n_rb, int L, int Hl, int D, int Lp, cudaStream_t stream);

// Row tables (-LSE*log2(e), -Delta) of one dilated-attention backward launch,
// gathered from the final LSE and Delta of every row ([B*S*Hq]); see
// usp_elementwise.cu.
cudaError_t launch_dilated_tables(const float* lse, const float* delta_all, float* lse2_t, float* delta_t,
                                  const FwdSub& sb, int Lp, cudaStream_t stream);
// fp32 -> bf16 of n elements (n % 4 == 0, 16-byte aligned).
cudaError_t launch_f32_to_bf16(const float* x, void* y, long long n, cudaStream_t stream);

struct BwdLaunch {
  AttnGeom g;
  CUtensorMap tm_q, tm_k, tm_v, tm_do;
  const float* lse2;   // [n_ranks*B*Hq_l][Lp]: -LSE*log2(e), -inf on padding rows
  const float* delta;  // [n_ranks*B*Hq_l][Lp]: -Delta, 0 on padding rows
  int Lp;
  void* dq;            // bf16, q layout (written by the query-major kernel)
  float* dk;           // fp32, k layout
  float* dv;           // fp32, v layout
  void* dk_bf16;       // mesh mode only: when set, dK and dV are written as bf16 here (k, v layout)
  void* dv_bf16;       // instead of dk, dv
  int* status;
  unsigned long long wait_ns;
  MaskArgs mask;       // masked variant when mask.bm or mask.cu is set
  // local mode: one rank (loc_i, loc_u) of a real mesh at ring step loc_t, whose
  // KV block belongs to ring rank loc_j = (loc_i - loc_t) mod P_r; its own buffers
  // (B in dim 4); dK, dV and the fp32 dq_acc are accumulated into
  int local, loc_i, loc_u, loc_t, loc_j;
  float* dq_acc;       // local and sub-problem modes: fp32 dQ accumulator
  FwdSub sub;          // sub-problem mode (dilated attention) when sub.active
};
cudaError_t launch_attn_bwd(const BwdLaunch& a, cudaStream_t stream);     // dK, dV (key-major)
cudaError_t launch_attn_bwd_dq(const BwdLaunch& a, cudaStream_t stream);  // dQ (query-major)

// LongNet dilated attention of one (w, r) pair over B sequences of S tokens
// (global layout [B][S][H][D]), every head offset (usp_dilated.cu): the forward
// folds the pair's result into the running fp32 (O, LSE); the backward adds the
// pair's dQ (into the fp32 dq_acc), dK and dV (fp32), with the final LSE and
// Delta of every row and two row-table buffers of dilated_pair_table_floats
// floats each (kSideStreams slots: the offsets of a pair write disjoint rows,
// o + tau r of each segment, so their launches run on side streams at the same
// time). With `first` (only for r = 1, whose launch covers every row and head)
// the forward writes the running result instead of folding, so it needs no
// initialisation. usp_status.
int dilated_fold_pair(const void* q, const void* k, const void* v, int B, int S, int Hq, int Hkv, int D, int causal,
                      int w, int r, float* o_run, float* lse_run, int* status, cudaStream_t st, int first = 0);
size_t dilated_pair_table_floats(int B, int S, int Hq, int w, int r);
int dilated_bwd_pair(const void* q, const void* k, const void* v, const void* dO, const float* lse,
                     const float* delta_all, float* dq_acc, float* dK, float* dV, float* lse2_t, float* delta_t, int B,
                     int S, int Hq, int Hkv, int D, int causal, int w, int r, int* status, cudaStream_t st,
                     int first = 0);

}  // namespace usp
