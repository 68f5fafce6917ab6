// usp_attn_bwd.cu -- backward of the blockwise USP attention on sm_100a: the
// key-major half (dK, dV). The query-major half (dQ) is usp_attn_bwd_dq.cu.
//
// What it computes (the gradient of the forward's exact attention; the pages
// give no formula, these are the derivatives of softmax attention): with P
// recomputed from the forward's final merged LSE,
//   P_ij = exp(scale q_i.k_j - LSE_i),   dP = dO V^T,   Delta_i = sum_d dO_id O_id,
//   dS = P o (dP - Delta),   dK = scale dS^T Q,   dV = P^T dO,
// with dK/dV summed over the q-heads of a GQA group and over every ring rank's
// queries (in the ring algorithm dK/dV travel around the ring with K/V).
//
// CTA = one 128-key tile of one kv-head of one head-sharded rank (the ring's KV
// chunk owner); it walks the q-heads of the group, the ring ranks whose queries
// see the tile and their 128-row query tiles ("steps"). 320 threads:
//   warp 0      TMA: K, V once; per step Q, dO (2 stages) and 128 LSE/Delta values;
//               it alone walks the steps and publishes one descriptor per step.
//   warp 1      TMEM allocator + UMMA issuer, per step k:
//                 S^T  = K Q^T     -> TMEM [0,128)     (M = keys, N = queries)
//                 dP^T = V dO^T    -> TMEM [128,256)   (overlaps the P^T phase below)
//                 dV  += P^T dO    -> TMEM [256,256+D) (A = P^T read from TMEM)
//                 dK  += dS^T Q    -> TMEM [384,384+D) (A = dS^T read from TMEM)
//               Order per step: dV(k), S^T(k+1) (as soon as dV has read P^T from
//               its columns), dK(k), dP^T(k+1) (once dK has read dS^T), so that
//               the P^T phase of step k+1 overlaps dK(k) and dP^T(k+1).
//   warps 2..9  two warpgroups; warpgroup c owns query columns [64c, 64c+64).
//               Thread = key row, in two phases per step: P^T as bf16 over the S^T
//               columns as soon as S^T lands (dV starts on it while dP^T is still
//               in flight), then dS^T over the dP^T columns (dK starts on it). At
//               the end dK and dV rows are written out in fp32 (added to the
//               buffers in the local and sub-problem modes) or, in the mesh mode
//               when asked, rounded once to bf16.
// Every wait is bounded (usp_ptx.cuh).
#include <math.h>

#include "usp_attn_common.cuh"
#include "usp_internal.h"
#include "usp_ptx.cuh"

namespace usp {
namespace {

constexpr int kThreadsBwd = 320;
constexpr int kComputeThreads = 256;
constexpr uint32_t kTmemColsBwd = 512;
constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 384;
constexpr int kPolyPer8 = 2;  // key pairs (of every 8) whose exp2 runs on the FMA pipe

template <int D>
struct BwdCfg {
  static constexpr int kPanels = D / 64;
  static constexpr int kPanelBytes = 128 * 128;
  static constexpr int kTileBytes = kPanels * kPanelBytes;
  static constexpr int kStages = 2;
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kTileBytes;
  static constexpr int kOffQ = 2 * kTileBytes;
  static constexpr int kOffDO = kOffQ + kStages * kTileBytes;
  static constexpr int kOffRow = kOffDO + kStages * kTileBytes;  // per stage: -LSE*log2e [128], -Delta [128]
  static constexpr int kOffBar = kOffRow + kStages * 1024;
  // No alignment slack: the kernel requires (and checks) a 1024-byte aligned dynamic shared memory base.
  static constexpr int kSmemBytes = kOffBar + 256;
};

struct BwdArgs {
  Geo g;
  const float* lse2;   // [n_ranks*B*Hq_l][Lp]: -LSE * log2(e)
  const float* delta;  // [n_ranks*B*Hq_l][Lp]: -Delta
  int Lp;
  float* dk;           // fp32 [n_ranks][B][L][Hkv_l][D]
  float* dv;
  void* dk_bf16;       // mesh mode: when set, dK and dV are written here as bf16 instead
  void* dv_bf16;
  int* status;
  unsigned long long wait_ns;
  int loc_i, loc_u, loc_j;  // local mode: query rank (i, u), KV block of ring rank j
  FwdSub sub;               // sub-problem mode (dilated attention): see usp_internal.h
};

struct BwdBars {
  uint64_t kv_full;
  uint64_t qd_full[2], qd_empty[2];
  uint64_t s_full, dp_full, p_full, ds_full, p_used, ds_used, drain;
  // Step descriptors published by the producer with qd_full of that step:
  // {q-head in group (-1 = no more steps), ring rank i, query tile m, tile kind}.
  int step[4][4];
  uint32_t tmem_base;
  int abort_flag;
};

enum : int {
  kSiteBKv = 0x201, kSiteBQdEmpty = 0x202, kSiteBQd = 0x211, kSiteBDsUsed = 0x212, kSiteBP = 0x213,
  kSiteBPUsed = 0x214, kSiteBDs = 0x215, kSiteBSt = 0x221, kSiteBDp = 0x222, kSiteBQdC = 0x223, kSiteBEpi = 0x224,
  kSiteBAlign = 0x2FF
};

// Query steps of one key tile: q-head hh of the group, ring rank i, query tile m.
struct QWalk {
  int hh, t, m, i, kind;
  bool valid;
};

template <bool kPlain = false>
__device__ __forceinline__ int classify_q(const Geo& g, int i, int m, int kmin, int kmax) {
  const int q0 = m * kBM;
  int qmin, qmax;
  qpos_range<kPlain>(g, i, q0, q0 + kBM, qmin, qmax);
  // Padded query columns need no mask: their LSE is +inf, so P = 0 there.
  if (g.causal && qmax < kmin) return kSkip;
  if (!g.causal || qmin >= kmax) return kFull;
  return kMasked;
}

// Masked variant: the causal kind narrowed by the block / document masks (the
// query tile of ring rank i, tile m, head hh of the group of kv-head gl).
struct MaskedQ {
  const Geo& g;
  int b, u, gl, kmin, kmax;
  __device__ __forceinline__ int operator()(int hh, int i, int m) const {
    const int kind = classify_q(g, i, m, kmin, kmax);
    int qmin, qmax;
    pos_range(g, i, m * kBM, m * kBM + kBM, qmin, qmax);
    return mask_tile(g.mask, kind, b, u * g.Hq_l + gl * g.G + hh, qmin, qmax, kmin, kmax);
  }
};

// Steps t in [t_lo, t_hi) of the walk: all ring ranks i = (j + t) mod P_r, or
// in the local mode the one rank that computes.
// In the sub-problem mode (kPlain) only the q-heads of the group that belong to
// the launch (hbase + hh congruent to hoff mod hstep) are walked.
template <bool kMask, bool kPlain = false>
__device__ __forceinline__ void qwalk_settle(const Geo& g, int j, int kmin, int kmax, QWalk& w, const MaskedQ& mq,
                                             int t_lo, int t_hi, int hbase = 0, int hoff = 0, int hstep = 1) {
  while (w.hh < g.G) {
    if (kPlain && (hbase + w.hh - hoff) % hstep != 0) {
      ++w.hh;
      continue;
    }
    while (w.t < t_hi) {
      w.i = (j + w.t) % g.P_r;
      while (w.m < g.n_qtiles) {
        w.kind = kMask ? mq(w.hh, w.i, w.m) : classify_q<kPlain>(g, w.i, w.m, kmin, kmax);
        if (w.kind != kSkip) {
          w.valid = true;
          return;
        }
        ++w.m;
      }
      ++w.t;
      w.m = 0;
    }
    ++w.hh;
    w.t = t_lo;
  }
  w.valid = false;
}

template <bool kMask, bool kPlain = false>
__device__ __forceinline__ QWalk qwalk_begin(const Geo& g, int j, int kmin, int kmax, const MaskedQ& mq, int t_lo,
                                             int t_hi, int hbase = 0, int hoff = 0, int hstep = 1) {
  QWalk w{0, t_lo, 0, 0, 0, false};
  qwalk_settle<kMask, kPlain>(g, j, kmin, kmax, w, mq, t_lo, t_hi, hbase, hoff, hstep);
  return w;
}

template <bool kMask, bool kPlain = false>
__device__ __forceinline__ void qwalk_next(const Geo& g, int j, int kmin, int kmax, QWalk& w, const MaskedQ& mq,
                                           int t_lo, int t_hi, int hbase = 0, int hoff = 0, int hstep = 1) {
  ++w.m;
  qwalk_settle<kMask, kPlain>(g, j, kmin, kmax, w, mq, t_lo, t_hi, hbase, hoff, hstep);
}

enum : int { kModeUsp = 0, kModeSub = 1, kModeLocal = 2 };

// kMode: kModeUsp -- every virtual rank of the mesh; kModeLocal -- ONE rank of a
// real multi-GPU mesh: the KV block of ring rank loc_j it holds (its own
// buffers, [B][L][Hkv/P_u][D]) against the queries of rank (loc_i, loc_u) only,
// dK and dV ADDED to the given fp32 buffers (the gradients travelling with the
// block around the ring); kModeSub -- the one-rank problems of a dilated
// attention launch (a (w, r) pair and head offset; strided tensor maps), dK and
// dV ADDED at the kept rows' original positions.
template <int D, bool kMask, int kMode>
__global__ void __launch_bounds__(kThreadsBwd, 1)
    attn_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    const BwdArgs a) {
  constexpr bool kLocal = kMode == kModeLocal;
  constexpr bool kSub = kMode == kModeSub;
  using C = BwdCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_addr(smem_raw) & 1023u) {  // the swizzled tiles need 1024-byte alignment
    if (threadIdx.x == 0) atomicCAS(a.status, 0, kSiteBAlign);
    return;
  }
  uint8_t* smem = smem_raw;
  BwdBars* bars = reinterpret_cast<BwdBars*>(smem + C::kOffBar);
  static_assert(sizeof(BwdBars) <= 256, "barrier block");
  uint8_t* sK = smem + C::kOffK;
  uint8_t* sV = smem + C::kOffV;
  uint8_t* sQ = smem + C::kOffQ;
  uint8_t* sDO = smem + C::kOffDO;
  float* sRow = reinterpret_cast<float*>(smem + C::kOffRow);

  const Geo& g = a.g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // Work item: CTAs of one (b, Ulysses rank, kv-head) run together; inside it,
  // key tiles in increasing original position (the causally heaviest first).
  int gl, u, b, j, n, prob = 0;
  if constexpr (kSub) {  // work item: (problem, kv-head of the launch, key tile)
    int wi = blockIdx.x;
    n = wi % g.n_ktiles;
    wi /= g.n_ktiles;
    gl = a.sub.kv0 + (wi % a.sub.n_kv) * a.sub.kv_step;
    prob = wi / a.sub.n_kv;
    u = b = j = 0;
  } else if constexpr (kLocal) {
    int wi = blockIdx.x;
    n = wi % g.n_ktiles;
    wi /= g.n_ktiles;
    gl = wi % g.Hkv_l;
    b = wi / g.Hkv_l;
    u = a.loc_u;
    j = a.loc_j;
  } else {
    const int n_kt = g.P_r * g.n_ktiles;
    int wi = blockIdx.x;
    const int order = wi % n_kt;
    wi /= n_kt;
    gl = wi % g.Hkv_l;
    wi /= g.Hkv_l;
    u = wi % g.P_u;
    b = wi / g.P_u;
    tile_in_position_order(g, order, j, n);
  }
  const int jrank = (kLocal || kSub) ? 0 : j * g.P_u + u;  // local buffers hold one rank
  // ring steps walked: every rank's queries, or those of the one local rank
  const int t_lo = kLocal ? (a.loc_i - j + g.P_r) % g.P_r : 0;
  const int t_hi = kLocal ? t_lo + 1 : g.P_r;
  const int k0 = n * kBN;
  int kmin, kmax;
  pos_range<kSub>(g, j, k0, k0 + kBN, kmin, kmax);

  if (threadIdx.x == 0) {
    bars->abort_flag = *reinterpret_cast<volatile int*>(a.status) != 0;
    mbar_init(&bars->kv_full, 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&bars->qd_full[s], 1);
      mbar_init(&bars->qd_empty[s], 1);
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->dp_full, 1);
    mbar_init(&bars->p_full, kComputeThreads / 32);  // one arrival per compute warp
    mbar_init(&bars->ds_full, kComputeThreads / 32);
    mbar_init(&bars->p_used, 1);
    mbar_init(&bars->ds_used, 1);
    mbar_init(&bars->drain, 1);
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(&bars->tmem_base, kTmemColsBwd);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const WaitCtl w{&bars->abort_flag, a.status, a.wait_ns};
  const bool skip = bars->abort_flag != 0;

  if (skip) {
    // nothing issued, nothing to drain
  } else if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    // The whole warp walks the steps (the same values in every lane); one elected
    // lane issues each copy and barrier operation.
    {
      if (lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        tma_prefetch_desc(&tm_do);
      }
      __syncwarp();
      const int krb = kSub ? prob : jrank * g.B + b;
      mbar_expect_tx_w(&bars->kv_full, 2 * C::kTileBytes);
      for (int p = 0; p < C::kPanels; ++p) {
        tma_load_4d_w(&tm_k, &bars->kv_full, sK + p * C::kPanelBytes, p * 64, gl, k0, krb);
        tma_load_4d_w(&tm_v, &bars->kv_full, sV + p * C::kPanelBytes, p * 64, gl, k0, krb);
      }
      int issued = 0;
      const MaskedQ mq{g, b, u, gl, kmin, kmax};
      // sub-problem mode: the launch's q-heads are a.sub.h0 + k * a.sub.h_step
      QWalk qw = qwalk_begin<kMask, kSub>(g, j, kmin, kmax, mq, t_lo, t_hi, gl * g.G, a.sub.h0, a.sub.h_step);
      while (true) {
        const int s = issued % C::kStages;
        if (issued >= C::kStages &&
            !mbar_wait_w(&bars->qd_empty[s], ((issued / C::kStages) - 1) & 1, w, kSiteBQdEmpty))
          break;
        int* slot = bars->step[issued & 3];
        if (!qw.valid) {  // publish the end of the walk on this stage's barrier
          if (lane == 0) slot[0] = -1;
          __syncwarp();
          mbar_arrive_w(&bars->qd_full[s]);
          break;
        }
        if (lane == 0) {
          slot[0] = qw.hh;
          slot[1] = qw.i;
          slot[2] = qw.m;
          slot[3] = qw.kind;
        }
        __syncwarp();
        const int h = gl * g.G + qw.hh;
        const int qrb = kSub ? prob : kLocal ? b : (qw.i * g.P_u + u) * g.B + b;
        const int q0 = qw.m * kBM;
        mbar_expect_tx_w(&bars->qd_full[s], 2 * C::kTileBytes + 1024);
        for (int p = 0; p < C::kPanels; ++p) {
          tma_load_4d_w(&tm_q, &bars->qd_full[s], sQ + s * C::kTileBytes + p * C::kPanelBytes, p * 64, h, q0, qrb);
          tma_load_4d_w(&tm_do, &bars->qd_full[s], sDO + s * C::kTileBytes + p * C::kPanelBytes, p * 64, h, q0,
                        qrb);
        }
        // row tables: per (rank, head), or per (problem, launch head) in the sub-problem mode
        const size_t rowbase =
            kSub ? (static_cast<size_t>(prob) * a.sub.n_heads + (h - a.sub.h0) / a.sub.h_step) * a.Lp + q0
                 : (static_cast<size_t>(qrb) * g.Hq_l + h) * a.Lp + q0;
        bulk_load_1d_w(sRow + s * 256, a.lse2 + rowbase, 512, &bars->qd_full[s]);
        bulk_load_1d_w(sRow + s * 256 + 128, a.delta + rowbase, 512, &bars->qd_full[s]);
        ++issued;
        qwalk_next<kMask, kSub>(g, j, kmin, kmax, qw, mq, t_lo, t_hi, gl * g.G, a.sub.h0, a.sub.h_step);
      }
      if (*reinterpret_cast<volatile int*>(&bars->abort_flag)) {
        mbar_wait_drain(&bars->kv_full, 0, a.wait_ns);
        for (int it = issued - C::kStages < 0 ? 0 : issued - C::kStages; it < issued; ++it)
          mbar_wait_drain(&bars->qd_full[it % C::kStages], (it / C::kStages) & 1, a.wait_ns);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ UMMA issuer
    // The whole warp runs this loop; one elected lane issues each UMMA/commit.
    {
      constexpr uint32_t kIdSS = idesc_bf16_f32(128, 128, 0, 0);  // both K-major
      constexpr uint32_t kIdKM = idesc_bf16_f32(128, D, 0, 1);    // A K-major, B MN-major
      // tile-base descriptors; a byte offset inside shared memory adds (offset >> 4)
      const uint64_t dK0 = sdesc_sw128(smem_addr(sK), 16, 1024), dV0 = sdesc_sw128(smem_addr(sV), 16, 1024);
      const uint64_t dQ0 = sdesc_sw128(smem_addr(sQ), 16, 1024), dDO0 = sdesc_sw128(smem_addr(sDO), 16, 1024);
      const uint64_t dQmn = sdesc_sw128(smem_addr(sQ), C::kPanelBytes, 1024);
      const uint64_t dDOmn = sdesc_sw128(smem_addr(sDO), C::kPanelBytes, 1024);
      auto issue_xt = [&](uint32_t col, uint64_t a0, uint64_t b0, int s) {  // X^T = A B_s^T (S^T or dP^T)
        const uint64_t bd = b0 + ((s * C::kTileBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * C::kPanelBytes + (kk & 3) * 32) >> 4;
          umma_bf16_w(tmem + col, a0 + off, bd + off, kIdSS, kk > 0 ? 1u : 0u);
        }
      };
      // acc += X^T Y_s with X^T packed in TMEM (warpgroup c's 64 queries at columns
      // 64c .. 64c+31 of its block) and Y_s (Q or dO of stage s) read MN-major
      auto issue_acc = [&](uint32_t acc, uint32_t xcol, uint64_t y0, int s, bool first) {
        const uint64_t yd = y0 + ((s * C::kTileBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < kBM / 16; ++kk) {
          const uint32_t pcol = (kk < 4 ? 0u : 64u) + (kk & 3) * 8;
          umma_bf16_tmem_a_w(tmem + acc, tmem + xcol + pcol, yd + ((kk * 16 * 128) >> 4), kIdKM,
                             (!first || kk > 0) ? 1u : 0u);
        }
      };
      bool ok = mbar_wait_w(&bars->kv_full, 0, w, kSiteBKv);
      bool issued_any = false;
      bool have = false;
      int k = 0;
      if (ok) ok = mbar_wait_w(&bars->qd_full[0], 0, w, kSiteBQd);
      if (ok) {
        have = bars->step[0][0] >= 0;
        if (have) {
          tc_fence_after();
          issue_xt(kColS, dK0, dQ0, 0);
          umma_commit_w(&bars->s_full);
          issue_xt(kColDP, dV0, dDO0, 0);
          umma_commit_w(&bars->dp_full);
          issued_any = true;
        }
      }
      for (; ok && have; ++k) {
        const int s = k % C::kStages;
        const int s1 = (k + 1) % C::kStages;
        if (!mbar_wait_w(&bars->p_full, k & 1, w, kSiteBP)) { ok = false; break; }
        tc_fence_after();
        issue_acc(kColDV, kColS, dDOmn, s, k == 0);  // dV += P^T dO, K = 128 queries
        umma_commit_w(&bars->p_used);
        if (!mbar_wait_w(&bars->qd_full[s1], ((k + 1) / C::kStages) & 1, w, kSiteBQd)) { ok = false; break; }
        have = bars->step[(k + 1) & 3][0] >= 0;
        // S^T of the next step as soon as dV has read P^T from its columns, so that the
        // P^T phase of the next step overlaps dK and dP^T
        if (have) {
          if (!mbar_wait_w(&bars->p_used, k & 1, w, kSiteBPUsed)) { ok = false; break; }
          tc_fence_after();
          issue_xt(kColS, dK0, dQ0, s1);
          umma_commit_w(&bars->s_full);
        }
        if (!mbar_wait_w(&bars->ds_full, k & 1, w, kSiteBDs)) { ok = false; break; }
        tc_fence_after();
        issue_acc(kColDK, kColDP, dQmn, s, k == 0);  // dK += dS^T Q, K = 128 queries
        umma_commit_w(&bars->ds_used);
        umma_commit_w(&bars->qd_empty[s]);  // this step's Q/dO stage is free once these UMMAs land
        if (!have) break;
        // dP^T of the next step overwrites the dS^T that dK reads
        if (!mbar_wait_w(&bars->ds_used, k & 1, w, kSiteBDsUsed)) { ok = false; break; }
        tc_fence_after();
        issue_xt(kColDP, dV0, dDO0, s1);
        umma_commit_w(&bars->dp_full);
      }
      if (!ok && issued_any) {
        umma_commit_w(&bars->drain);
        mbar_wait_drain(&bars->drain, 0, a.wait_ns);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ compute warps
    const int cw = warp - 2;       // 0..7
    const int wg = cw >> 2;        // warpgroup: query columns [64 wg, 64 wg + 64)
    const int wq = warp & 3;       // TMEM lane quarter
    const int row = wq * 32 + lane;  // key row of S^T/dP^T/dK/dV; query row of the dQ tile
    const uint32_t trow = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const int tau_k = k0 + row;
    const int pos_k = tau_k < g.L ? token_pos<kSub>(g, j, tau_k) : INT_MAX;  // padding keys see no query
    int doc_lo = 0, doc_hi = INT_MAX;  // the key's document [lo, hi) (masked variant)
    if constexpr (kMask) doc_span(g.mask, pos_k, doc_lo, doc_hi);
    const bool aligned = (g.c % kBM) == 0;
    const int cbase = wg * 64;
    bool ok = true;
    int k = 0;
    for (;; ++k) {
      const int s = k % C::kStages;
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->qd_full[s], (k / C::kStages) & 1, w, kSiteBQdC));
      if (!ok) break;
      const int* slot = bars->step[k & 3];
      const int st_hh = slot[0];
      if (st_hh < 0) break;
      const int st_i = slot[1], st_m = slot[2], st_kind = slot[3];
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->s_full, k & 1, w, kSiteBSt));
      if (!ok) break;
      tc_fence_after();
      const float* nlse2 = sRow + s * 256;  // -LSE*log2(e) of the 128 query rows
      const float* ndl = nlse2 + 128;         // -Delta of the 128 query rows
      const int q0 = st_m * kBM;
      if (st_kind == kMasked) {
        // causal: rewrite S^T of this key row to -inf where the query does not see
        // the key, so the main pass carries no masking (P = 0 there)
        int lo = pos_k == INT_MAX ? kBM : pos_k - qtoken_pos<kSub>(g, st_i, q0);  // aligned: cols >= lo see it
        int hi_c = kBM;                                                      // and cols < hi_c
        if constexpr (kMask) {
          // masked variant (tiles contiguous): the key's document bounds the columns too
          const int qpos0 = qtoken_pos<kSub>(g, st_i, q0);
          if (!g.causal && pos_k != INT_MAX) lo = 0;
          if (pos_k != INT_MAX) {
            lo = max(lo, doc_lo - qpos0);
            if (doc_hi != INT_MAX) hi_c = doc_hi - qpos0;
          }
        }
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
          const int c0 = cbase + half * 32;
          uint32_t vis;  // bit c: query column c0 + c sees this key
          if (aligned) {
            const int nb = min(max(lo - c0, 0), 32);  // leading invisible columns
            vis = nb >= 32 ? 0u : (0xFFFFFFFFu << nb);
            if constexpr (kMask) {
              const int nt = min(max(hi_c - c0, 0), 32);  // columns below hi_c
              vis &= nt >= 32 ? 0xFFFFFFFFu : ((1u << nt) - 1u);
            }
          } else {
            vis = 0u;
            for (int c = 0; c < 32; ++c) {
              const int tq = q0 + c0 + c;
              if (tq < g.Lq && pos_k <= qtoken_pos<kSub>(g, st_i, tq)) vis |= 1u << c;
            }
          }
          uint32_t r[32];
          tmem_ld32(trow + kColS + c0, r);
          tmem_ld_wait();
          reg_fence32(r);
#pragma unroll
          for (int c = 0; c < 32; ++c)
            if (!((vis >> c) & 1u)) r[c] = 0xFF800000u;  // -inf
          tmem_st32(trow + kColS + c0, r);
        }
        tmem_st_wait();
      }
      // Phase 1 (while the tensor core computes dP^T): P^T = exp2(s*scale*log2e - LSE*log2e)
      // as bf16 over the S^T columns; the fp32 values stay in registers for dS.
      float2 pr[32];
      const float2 sl2 = make_float2(g.scale_log2, g.scale_log2);
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int c0 = cbase + half * 32;
        uint32_t rs[32];
        tmem_ld32(trow + kColS + c0, rs);
        tmem_ld_wait();
        reg_fence32(rs);
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          const float2 nl = *reinterpret_cast<const float2*>(nlse2 + c0 + c);  // smem broadcast
          const float2 x = ffma2(make_float2(__uint_as_float(rs[c]), __uint_as_float(rs[c + 1])), sl2, nl);
          // kPolyPer8 key pairs in every 8 take the polynomial exp2 on the FMA pipe,
          // which has room in this kernel while the MUFU bounds the P phase. A -inf
          // score gets ~2^-125 there instead of 0: a weight no dK/dV sum resolves.
          const float2 pv = ((c >> 1) % 8 < kPolyPer8) ? exp2_poly2(x)
                                                       : make_float2(ex2_approx(x.x), ex2_approx(x.y));
          pr[half * 16 + (c >> 1)] = pv;
          pk[c >> 1] = pack_bf16x2(pv.x, pv.y);
        }
        tmem_st16(trow + kColS + cbase + half * 16, pk);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive_warp(&bars->p_full);
      // Phase 2 (while the tensor core computes dV): dS^T = P^T o (dP^T - Delta) as
      // bf16 over the dP^T columns (without the softmax scale, applied to dK at the end).
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->dp_full, k & 1, w, kSiteBDp));
      if (!ok) break;
      tc_fence_after();
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int c0 = cbase + half * 32;
        uint32_t rp[32];
        tmem_ld32(trow + kColDP + c0, rp);
        tmem_ld_wait();
        reg_fence32(rp);
        uint32_t dk[16];
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          const float2 nd = *reinterpret_cast<const float2*>(ndl + c0 + c);
          const float2 ds = fmul2(pr[half * 16 + (c >> 1)],
                                  fadd2(make_float2(__uint_as_float(rp[c]), __uint_as_float(rp[c + 1])), nd));
          dk[c >> 1] = pack_bf16x2(ds.x, ds.y);
        }
        tmem_st16(trow + kColDP + cbase + half * 16, dk);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive_warp(&bars->ds_full);
    }
    // ------------------------------------------------------------ dK, dV epilogue
    // the last step's dK/dV UMMAs (and every earlier one) have landed once its ds_used arrives
    if (ok && k >= 1) ok = __all_sync(0xffffffffu, mbar_wait(&bars->ds_used, (k - 1) & 1, w, kSiteBEpi));
    // adding the gradients of a key tile that no query saw changes nothing: no read, no write
    const bool noop = k == 0 && (kLocal || (kSub && !a.sub.first));
    if (ok && !noop) {
      tc_fence_after();
      const bool store = tau_k < g.L;
      size_t kr;
      if constexpr (kSub) {  // the key's row in the dK/dV buffers (its original position, or a gathered row)
        const int pb = prob / a.sub.n_seg, ps = prob % a.sub.n_seg;
        kr = (static_cast<size_t>(pb) * a.sub.kS + static_cast<size_t>(ps) * a.sub.kw + a.sub.koff +
              static_cast<size_t>(store ? tau_k : 0) * a.sub.kstep) * a.sub.kH + gl;
      } else {
        kr = (static_cast<size_t>(jrank * g.B + b) * g.L + (store ? tau_k : 0)) * g.Hkv_l + gl;
      }
      // warpgroup wg writes columns [wg*D/2, wg*D/2 + D/2)
#pragma unroll
      for (int c0 = wg * (D / 2); c0 < (wg + 1) * (D / 2); c0 += 32) {
        uint32_t rk[32], rv[32];
        if (k >= 1) {
          tmem_ld32(trow + kColDK + c0, rk);
          tmem_ld32(trow + kColDV + c0, rv);
          tmem_ld_wait();
          reg_fence32(rk);
          reg_fence32(rv);
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) rk[c] = rv[c] = 0u;
        }
        if (store && !kLocal && !kSub && a.dk_bf16 != nullptr) {
          // the gradients in the inputs' type, rounded once from the fp32 sums
          uint4* dkp = reinterpret_cast<uint4*>(static_cast<uint16_t*>(a.dk_bf16) + kr * D + c0);
          uint4* dvp = reinterpret_cast<uint4*>(static_cast<uint16_t*>(a.dv_bf16) + kr * D + c0);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 hk, hv;
            hk.x = pack_bf16x2(__uint_as_float(rk[8 * q + 0]) * g.scale, __uint_as_float(rk[8 * q + 1]) * g.scale);
            hk.y = pack_bf16x2(__uint_as_float(rk[8 * q + 2]) * g.scale, __uint_as_float(rk[8 * q + 3]) * g.scale);
            hk.z = pack_bf16x2(__uint_as_float(rk[8 * q + 4]) * g.scale, __uint_as_float(rk[8 * q + 5]) * g.scale);
            hk.w = pack_bf16x2(__uint_as_float(rk[8 * q + 6]) * g.scale, __uint_as_float(rk[8 * q + 7]) * g.scale);
            hv.x = pack_bf16x2(__uint_as_float(rv[8 * q + 0]), __uint_as_float(rv[8 * q + 1]));
            hv.y = pack_bf16x2(__uint_as_float(rv[8 * q + 2]), __uint_as_float(rv[8 * q + 3]));
            hv.z = pack_bf16x2(__uint_as_float(rv[8 * q + 4]), __uint_as_float(rv[8 * q + 5]));
            hv.w = pack_bf16x2(__uint_as_float(rv[8 * q + 6]), __uint_as_float(rv[8 * q + 7]));
            dkp[q] = hk;
            dvp[q] = hv;
          }
        } else if (store) {
          float4* dkp = reinterpret_cast<float4*>(a.dk + kr * D + c0);
          float4* dvp = reinterpret_cast<float4*>(a.dv + kr * D + c0);
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            float4 nk = make_float4(__uint_as_float(rk[4 * q]) * g.scale, __uint_as_float(rk[4 * q + 1]) * g.scale,
                                    __uint_as_float(rk[4 * q + 2]) * g.scale, __uint_as_float(rk[4 * q + 3]) * g.scale);
            float4 nv = make_float4(__uint_as_float(rv[4 * q]), __uint_as_float(rv[4 * q + 1]),
                                    __uint_as_float(rv[4 * q + 2]), __uint_as_float(rv[4 * q + 3]));
            // add (travelling ring gradients; the pairs' sum, but for a dilated pair with r = 1
            // run first, which writes)
            if (kLocal || (kSub && !a.sub.first)) {
              const float4 ok_ = dkp[q], ov = dvp[q];
              nk = make_float4(nk.x + ok_.x, nk.y + ok_.y, nk.z + ok_.z, nk.w + ok_.w);
              nv = make_float4(nv.x + ov.x, nv.y + ov.y, nv.z + ov.z, nv.w + ov.w);
            }
            dkp[q] = nk;
            dvp[q] = nv;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemColsBwd);
  }
}

template <int D, bool kMask, int kMode>
cudaError_t launch_bwd_d(const BwdLaunch& L, cudaStream_t stream) {
  constexpr bool kLocal = kMode == kModeLocal;
  constexpr bool kSub = kMode == kModeSub;
  using C = BwdCfg<D>;
  static_assert(C::kSmemBytes <= 227 * 1024, "shared memory budget");
  cudaError_t e = cudaFuncSetAttribute(attn_bwd_kernel<D, kMask, kMode>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  BwdArgs a{};
  a.g = make_geo(L.g);
  a.g.mask = L.mask;
  a.lse2 = L.lse2;
  a.delta = L.delta;
  a.Lp = L.Lp;
  a.dk = L.dk;
  a.dv = L.dv;
  a.dk_bf16 = L.dk_bf16;
  a.dv_bf16 = L.dv_bf16;
  if ((kLocal || kSub) && (L.dk_bf16 != nullptr || L.dv_bf16 != nullptr)) return cudaErrorInvalidValue;
  if ((L.dk_bf16 == nullptr) != (L.dv_bf16 == nullptr)) return cudaErrorInvalidValue;
  a.status = L.status;
  a.wait_ns = L.wait_ns;
  a.loc_i = L.loc_i;
  a.loc_u = L.loc_u;
  a.loc_j = L.loc_j;
  a.sub = L.sub;
  if (kSub) {  // one-rank geometry of every problem (see the forward's sub-problem mode)
    if (a.sub.n_kv <= 0) {  // every kv head
      a.sub.kv0 = 0;
      a.sub.kv_step = 1;
      a.sub.n_kv = a.g.Hkv_l;
    }
    if (a.sub.kv0 < 0 || a.sub.kv_step < 1 || a.sub.kv0 + (a.sub.n_kv - 1) * a.sub.kv_step >= a.g.Hkv_l)
      return cudaErrorInvalidValue;
    a.g.P_u = a.g.P_r = a.g.P = a.g.n_ranks = 1;
    a.g.L = L.sub.L;
    a.g.c = kBN;
    a.g.Lq = L.sub.Lq;
    a.g.q_off = L.sub.q_off;
    a.g.n_qtiles = (L.sub.Lq + kBM - 1) / kBM;
    a.g.n_ktiles = (L.sub.L + kBN - 1) / kBN;
  }
  const long long blocks = kSub     ? static_cast<long long>(a.g.n_ktiles) * a.sub.n_kv * L.sub.n_prob
                           : kLocal ? static_cast<long long>(a.g.n_ktiles) * a.g.B * a.g.Hkv_l
                                    : static_cast<long long>(a.g.n_ktiles) * a.g.P_r * a.g.P_u * a.g.B * a.g.Hkv_l;
  if (blocks <= 0) return cudaSuccess;
  if (blocks > 0x7FFFFFFFLL) return cudaErrorInvalidConfiguration;
  attn_bwd_kernel<D, kMask, kMode><<<static_cast<unsigned>(blocks), kThreadsBwd, C::kSmemBytes, stream>>>(
      L.tm_q, L.tm_k, L.tm_v, L.tm_do, a);
  note_launch();
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_bwd(const BwdLaunch& L, cudaStream_t stream) {
  const bool masked = L.mask.bm != nullptr || L.mask.cu != nullptr;
  if (masked && (L.local || L.sub.active)) return cudaErrorInvalidValue;
  if (L.sub.active) {
    if (L.g.D == 128) return launch_bwd_d<128, false, kModeSub>(L, stream);
    if (L.g.D == 64) return launch_bwd_d<64, false, kModeSub>(L, stream);
    return cudaErrorInvalidValue;
  }
  if (L.local) {
    if (L.g.D == 128) return launch_bwd_d<128, false, kModeLocal>(L, stream);
    if (L.g.D == 64) return launch_bwd_d<64, false, kModeLocal>(L, stream);
    return cudaErrorInvalidValue;
  }
  if (masked) {
    if (L.g.D == 128) return launch_bwd_d<128, true, kModeUsp>(L, stream);
    if (L.g.D == 64) return launch_bwd_d<64, true, kModeUsp>(L, stream);
    return cudaErrorInvalidValue;
  }
  if (L.g.D == 128) return launch_bwd_d<128, false, kModeUsp>(L, stream);
  if (L.g.D == 64) return launch_bwd_d<64, false, kModeUsp>(L, stream);
  return cudaErrorInvalidValue;
}

}  // namespace usp
