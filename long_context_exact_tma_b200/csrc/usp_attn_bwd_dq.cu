// usp_attn_bwd_dq.cu -- backward of the blockwise USP attention on sm_100a: the
// query-major half (dQ). The key-major half (dK, dV) is usp_attn_bwd.cu.
//
// What it computes: for every query row i of every virtual rank, with P
// recomputed from the forward's final merged LSE (the derivative of exact
// softmax attention; the pages give no formula),
//   dQ_i = scale * sum_j P_ij (dP_ij - Delta_i) K_j,   dP_ij = dO_i . V_j,
// over the keys of every ring step (owner j = (i - t) mod P_r), walked in the
// same order and with the same causal mask as the forward. dQ accumulates in
// TMEM across the whole walk and is written once, as bf16: no cross-CTA
// reduction, at the price of recomputing S and dP (which the key-major half
// also computes).
//
// CTA = one 128-row query tile of one (rank, batch, head); 320 threads:
//   warp 0      TMA: Q and dO once, K tiles into 3 stages, V tiles into 2; it
//               alone walks the key tiles and publishes one descriptor per tile.
//   warp 1      TMEM allocator + UMMA issuer, per key tile t:
//                 S_t  = Q K^T     -> TMEM [128 (t&1), +128)   (double buffered)
//                 dP_t = dO V^T    -> TMEM [256, 384)
//                 dQ  += dS_t K    -> TMEM [384, 384+D)  (A = dS_t read from TMEM)
//               S_{t+1} and dP_{t+1} are issued before dQ_t, so the next tile's
//               scores are ready when the warpgroups finish this one.
//   warps 2..9  two warpgroups; warpgroup c owns key columns [64c, 64c+64).
//               Thread = query row: dS = exp2(S*scale*log2e - LSE*log2e) o (dP - Delta)
//               as bf16, packed into TMEM over the S columns it came from.
// Every wait is bounded (usp_ptx.cuh).
#include <math.h>

#include "usp_attn_common.cuh"
#include "usp_internal.h"
#include "usp_ptx.cuh"

namespace usp {
namespace {

constexpr int kThreadsDq = 320;
constexpr int kComputeDq = 256;
constexpr uint32_t kTmemColsDq = 512;
constexpr uint32_t kColDPq = 256, kColDQ = 384;
__host__ __device__ constexpr uint32_t col_sq(int b) { return 128u * b; }

template <int D>
struct DqCfg {
  static constexpr int kPanels = D / 64;
  static constexpr int kPanelBytes = 128 * 128;
  static constexpr int kTileBytes = kPanels * kPanelBytes;
  static constexpr int kKStages = 3;
  static constexpr int kVStages = 2;
  static constexpr int kOffQ = 0;
  static constexpr int kOffDO = kTileBytes;
  static constexpr int kOffK = 2 * kTileBytes;
  static constexpr int kOffV = kOffK + kKStages * kTileBytes;
  static constexpr int kOffBar = kOffV + kVStages * kTileBytes;
  // No alignment slack: the kernel requires (and checks) a 1024-byte aligned dynamic shared memory base.
  static constexpr int kSmemBytes = kOffBar + 256;
};

struct DqArgs {
  Geo g;
  const float* nlse2;   // [n_ranks*B*Hq_l][Lp]: -LSE * log2(e) (-inf on padding rows)
  const float* ndelta;  // [n_ranks*B*Hq_l][Lp]: -Delta (0 on padding rows)
  int Lp;
  __nv_bfloat16* dq;    // bf16 [n_ranks][B][L][Hq_l][D]
  float* dq_acc;        // local mode: fp32 [B][L][Hq_l][D], this step's dQ is added to it
  int loc_i, loc_u, loc_t;  // local mode: the rank (i, u) and its ring step t
  FwdSub sub;               // sub-problem mode (dilated attention): see usp_internal.h
  int* status;
  unsigned long long wait_ns;
};

struct DqBars {
  uint64_t q_full;
  uint64_t k_full[3], k_empty[3], v_full[2], v_empty[2];
  uint64_t s_full[2], dp_full, dp_free, ds_full, dq_done[2], drain;
  // Key-tile descriptors published by the producer with k_full of that tile:
  // {1, or -1 = no more tiles; ring rank j of the key owner; key tile n; tile kind}.
  int step[4][4];
  uint32_t tmem_base;
  int abort_flag;
};

enum : int {
  kSiteQQ = 0x301, kSiteQKEmpty = 0x302, kSiteQVEmpty = 0x303, kSiteQK = 0x311, kSiteQV = 0x312,
  kSiteQDpFree = 0x313, kSiteQDs = 0x314, kSiteQDqDone = 0x315, kSiteQKs = 0x321, kSiteQS = 0x322,
  kSiteQDp = 0x323, kSiteQEpi = 0x324, kSiteQAlign = 0x3FF
};

// kLocal: ONE rank (loc_i, loc_u) of a real multi-GPU mesh at ring step loc_t:
// its own Q and dO against the KV block it holds (owner (i - t) mod P_r), its
// own buffers ([B][L][H/P_u][D]); dQ is ADDED to the fp32 dq_acc.
enum : int { kModeUsp = 0, kModeSub = 1, kModeLocal = 2 };

// kModeSub: the one-rank problems of a dilated attention launch (a (w, r) pair
// and head offset, strided tensor maps); dQ is ADDED to the fp32 dq_acc at the
// kept rows' original positions.
template <int D, bool kMask, int kMode>
__global__ void __launch_bounds__(kThreadsDq, 1)
    attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                       const DqArgs a) {
  constexpr bool kLocal = kMode == kModeLocal;
  constexpr bool kSub = kMode == kModeSub;
  using C = DqCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_addr(smem_raw) & 1023u) {  // the swizzled tiles need 1024-byte alignment
    if (threadIdx.x == 0) atomicCAS(a.status, 0, kSiteQAlign);
    return;
  }
  uint8_t* smem = smem_raw;
  DqBars* bars = reinterpret_cast<DqBars*>(smem + C::kOffBar);
  static_assert(sizeof(DqBars) <= 256, "barrier block");
  uint8_t* sQ = smem + C::kOffQ;
  uint8_t* sDO = smem + C::kOffDO;
  uint8_t* sK = smem + C::kOffK;
  uint8_t* sV = smem + C::kOffV;

  const Geo& g = a.g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // Work item: CTAs of one (b, Ulysses rank, head) run together so that its K/V
  // stay in L2; inside it, query tiles in decreasing original position.
  int h, u, b, i, m, prob = 0;
  if constexpr (kSub) {  // work item: (problem, launch head, query tile), heaviest first
    int wi = blockIdx.x;
    m = g.n_qtiles - 1 - wi % g.n_qtiles;
    wi /= g.n_qtiles;
    h = a.sub.h0 + (wi % a.sub.n_heads) * a.sub.h_step;
    prob = wi / a.sub.n_heads;
    u = b = i = 0;
  } else if constexpr (kLocal) {
    int wi = blockIdx.x;
    m = g.n_qtiles - 1 - wi % g.n_qtiles;
    wi /= g.n_qtiles;
    h = wi % g.Hq_l;
    b = wi / g.Hq_l;
    i = a.loc_i;
    u = a.loc_u;
  } else {
    const int n_qt = g.P_r * g.n_qtiles;
    int wi = blockIdx.x;
    const int order = n_qt - 1 - wi % n_qt;
    wi /= n_qt;
    h = wi % g.Hq_l;
    wi /= g.Hq_l;
    u = wi % g.P_u;
    b = wi / g.P_u;
    tile_in_position_order(g, order, i, m);
  }
  const int rank = (kLocal || kSub) ? 0 : i * g.P_u + u;  // local buffers hold one rank
  // ring steps walked: all of them, or the local rank's one step
  const int t_lo = kLocal ? a.loc_t : 0;
  const int t_hi = kLocal ? a.loc_t + 1 : g.P_r;
  const int kvh = h / g.G;
  const int q0 = m * kBM;

  if (threadIdx.x == 0) {
    bars->abort_flag = *reinterpret_cast<volatile int*>(a.status) != 0;
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < C::kKStages; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
    }
    for (int s = 0; s < C::kVStages; ++s) {
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->s_full[s], 1);
      mbar_init(&bars->dq_done[s], 1);
    }
    mbar_init(&bars->dp_full, 1);
    mbar_init(&bars->dp_free, kComputeDq / 32);  // one arrival per compute warp
    mbar_init(&bars->ds_full, kComputeDq / 32);
    mbar_init(&bars->drain, 1);
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(&bars->tmem_base, kTmemColsDq);
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
    // The whole warp walks the key tiles (the same values in every lane); one
    // elected lane issues each copy and barrier operation.
    {
      int qmin, qmax;
      qpos_range<kSub>(g, i, q0, q0 + kBM, qmin, qmax);
      // masked variant: the causal kind narrowed by the block / document masks
      auto kind_of = [&](int j, int n) {
        int kmin, kmax;
        pos_range(g, j, n * kBN, n * kBN + kBN, kmin, kmax);
        return mask_tile(g.mask, classify_tile(g, qmin, qmax, j, n), b, u * g.Hq_l + h, qmin, qmax, kmin, kmax);
      };
      KvWalk kw;
      if constexpr (kMask)
        kw = kv_walk_begin_by(g, i, t_lo, t_hi, kind_of);
      else
        kw = kv_walk_begin<kSub>(g, i, qmin, qmax, t_lo, t_hi);
      if (lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        tma_prefetch_desc(&tm_do);
      }
      __syncwarp();
      const int qrb = kSub ? prob : rank * g.B + b;
      mbar_expect_tx_w(&bars->q_full, 2 * C::kTileBytes);
      for (int p = 0; p < C::kPanels; ++p) {
        tma_load_4d_w(&tm_q, &bars->q_full, sQ + p * C::kPanelBytes, p * 64, h, q0, qrb);
        tma_load_4d_w(&tm_do, &bars->q_full, sDO + p * C::kPanelBytes, p * 64, h, q0, qrb);
      }
      int k_issued = 0, v_issued = 0;
      while (true) {
        const int it = k_issued;
        const int sk = it % C::kKStages, sv = it % C::kVStages;
        if (it >= C::kKStages &&
            !mbar_wait_w(&bars->k_empty[sk], ((it / C::kKStages) - 1) & 1, w, kSiteQKEmpty))
          break;
        int* slot = bars->step[it & 3];
        if (!kw.valid) {  // publish the end of the walk on this stage's barrier
          if (lane == 0) slot[0] = -1;
          __syncwarp();
          mbar_arrive_w(&bars->k_full[sk]);
          break;
        }
        if (lane == 0) {
          slot[0] = 1;
          slot[1] = kw.j;
          slot[2] = kw.n;
          slot[3] = kw.kind;
        }
        __syncwarp();
        const int krb = kSub ? prob : kLocal ? b : (kw.j * g.P_u + u) * g.B + b;
        mbar_expect_tx_w(&bars->k_full[sk], C::kTileBytes);
        for (int p = 0; p < C::kPanels; ++p)
          tma_load_4d_w(&tm_k, &bars->k_full[sk], sK + sk * C::kTileBytes + p * C::kPanelBytes, p * 64, kvh,
                        kw.n * kBN, krb);
        ++k_issued;
        if (it >= C::kVStages &&
            !mbar_wait_w(&bars->v_empty[sv], ((it / C::kVStages) - 1) & 1, w, kSiteQVEmpty))
          break;
        mbar_expect_tx_w(&bars->v_full[sv], C::kTileBytes);
        for (int p = 0; p < C::kPanels; ++p)
          tma_load_4d_w(&tm_v, &bars->v_full[sv], sV + sv * C::kTileBytes + p * C::kPanelBytes, p * 64, kvh,
                        kw.n * kBN, krb);
        ++v_issued;
        if constexpr (kMask)
          kv_walk_next_by(g, i, t_hi, kw, kind_of);
        else
          kv_walk_next<kSub>(g, i, qmin, qmax, t_hi, kw);
      }
      if (*reinterpret_cast<volatile int*>(&bars->abort_flag)) {
        // Let every copy this warp started land before the CTA exits.
        mbar_wait_drain(&bars->q_full, 0, a.wait_ns);
        for (int it = k_issued - C::kKStages < 0 ? 0 : k_issued - C::kKStages; it < k_issued; ++it)
          mbar_wait_drain(&bars->k_full[it % C::kKStages], (it / C::kKStages) & 1, a.wait_ns);
        for (int it = v_issued - C::kVStages < 0 ? 0 : v_issued - C::kVStages; it < v_issued; ++it)
          mbar_wait_drain(&bars->v_full[it % C::kVStages], (it / C::kVStages) & 1, a.wait_ns);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ UMMA issuer
    // The whole warp runs this loop; one elected lane issues each UMMA/commit.
    {
      constexpr uint32_t kIdSS = idesc_bf16_f32(128, 128, 0, 0);  // both K-major
      constexpr uint32_t kIdKM = idesc_bf16_f32(128, D, 0, 1);    // A (TMEM) K-major, B MN-major
      // tile-base descriptors; a byte offset inside shared memory adds (offset >> 4)
      const uint64_t dQ0 = sdesc_sw128(smem_addr(sQ), 16, 1024), dDO0 = sdesc_sw128(smem_addr(sDO), 16, 1024);
      const uint64_t dK0 = sdesc_sw128(smem_addr(sK), 16, 1024), dV0 = sdesc_sw128(smem_addr(sV), 16, 1024);
      const uint64_t dKmn = sdesc_sw128(smem_addr(sK), C::kPanelBytes, 1024);
      auto issue_s = [&](int it) {  // S_it = Q K_it^T into buffer it & 1
        const uint64_t kd = dK0 + (((it % C::kKStages) * C::kTileBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * C::kPanelBytes + (kk & 3) * 32) >> 4;
          umma_bf16_w(tmem + col_sq(it & 1), dQ0 + off, kd + off, kIdSS, kk > 0 ? 1u : 0u);
        }
        umma_commit_w(&bars->s_full[it & 1]);
      };
      auto issue_dp = [&](int it) {  // dP_it = dO V_it^T
        const uint64_t vd = dV0 + (((it % C::kVStages) * C::kTileBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * C::kPanelBytes + (kk & 3) * 32) >> 4;
          umma_bf16_w(tmem + kColDPq, dDO0 + off, vd + off, kIdSS, kk > 0 ? 1u : 0u);
        }
        umma_commit_w(&bars->dp_full);
        umma_commit_w(&bars->v_empty[it % C::kVStages]);
      };
      // tile `it` exists: wait for its K and read its descriptor
      auto has_tile = [&](int it, bool& ok_) -> bool {
        if (!mbar_wait_w(&bars->k_full[it % C::kKStages], (it / C::kKStages) & 1, w, kSiteQK)) {
          ok_ = false;
          return false;
        }
        return bars->step[it & 3][0] >= 0;
      };
      bool ok = true;
      bool issued_any = false;
      bool have0 = has_tile(0, ok);
      if (ok && have0) ok = mbar_wait_w(&bars->q_full, 0, w, kSiteQQ);
      bool have1 = false;
      if (ok && have0) {
        tc_fence_after();
        issue_s(0);
        issued_any = true;
        if ((ok = mbar_wait_w(&bars->v_full[0], 0, w, kSiteQV))) {
          tc_fence_after();
          issue_dp(0);
          have1 = has_tile(1, ok);
          if (ok && have1) issue_s(1);
        }
      }
      for (int it = 0; ok && have0; ++it) {
        // dP of the next tile as soon as this tile's dP has been read, ahead of dQ,
        // so that the warpgroups can start on the next tile while dQ accumulates
        if (have1) {
          if (!mbar_wait_w(&bars->v_full[(it + 1) % C::kVStages], ((it + 1) / C::kVStages) & 1, w, kSiteQV)) {
            ok = false;
            break;
          }
          if (!mbar_wait_w(&bars->dp_free, it & 1, w, kSiteQDpFree)) { ok = false; break; }
          tc_fence_after();
          issue_dp(it + 1);
        }
        if (!mbar_wait_w(&bars->ds_full, it & 1, w, kSiteQDs)) { ok = false; break; }
        tc_fence_after();
        const uint64_t kd = dKmn + (((it % C::kKStages) * C::kTileBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {  // dQ += dS K, K = 128 keys
          // warpgroup c packed its 64 keys at columns 64c .. 64c+31 of the S buffer
          const uint32_t pcol = col_sq(it & 1) + (kk < 4 ? 0u : 64u) + (kk & 3) * 8;
          umma_bf16_tmem_a_w(tmem + kColDQ, tmem + pcol, kd + ((kk * 16 * 128) >> 4), kIdKM,
                             (it > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit_w(&bars->dq_done[it & 1]);
        umma_commit_w(&bars->k_empty[it % C::kKStages]);
        if (!have1) break;
        // S of tile it+2 into this tile's S buffer once dQ has read dS from it
        const bool have2 = has_tile(it + 2, ok);
        if (!ok) break;
        if (have2) {
          if (!mbar_wait_w(&bars->dq_done[it & 1], (it >> 1) & 1, w, kSiteQDqDone)) { ok = false; break; }
          tc_fence_after();
          issue_s(it + 2);
        }
        have1 = have2;
      }
      if (!ok && issued_any) {
        umma_commit_w(&bars->drain);
        mbar_wait_drain(&bars->drain, 0, a.wait_ns);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ compute warps
    const int cw = warp - 2;
    const int wg = cw >> 2;          // warpgroup: key columns [64 wg, 64 wg + 64)
    const int wq = warp & 3;         // TMEM lane quarter
    const int row = wq * 32 + lane;  // query row of the tile
    const uint32_t trow = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const int cbase = wg * 64;
    const int tau_q = q0 + row;
    const int pos_q = tau_q < g.Lq ? qtoken_pos<kSub>(g, i, tau_q) : INT_MAX;
    const bool aligned = (g.c % kBN) == 0;
    int doc_lo = 0, doc_hi = INT_MAX;  // the row's document [lo, hi) (masked variant)
    if constexpr (kMask) doc_span(g.mask, pos_q, doc_lo, doc_hi);
    // row tables: per (rank, head), or per (problem, launch head) in the sub-problem mode
    const size_t tab =
        kSub ? (static_cast<size_t>(prob) * a.sub.n_heads + (h - a.sub.h0) / a.sub.h_step) * a.Lp + tau_q
             : (static_cast<size_t>(rank * g.B + b) * g.Hq_l + h) * a.Lp + tau_q;
    const float nl = __ldg(a.nlse2 + tab);   // -inf on padding rows: their P is 0
    const float nd = __ldg(a.ndelta + tab);
    const float2 sl2 = make_float2(g.scale_log2, g.scale_log2);
    const float2 nl2 = make_float2(nl, nl), nd2 = make_float2(nd, nd);
    bool ok = true;
    int it = 0;
    for (;; ++it) {
      ok = __all_sync(0xffffffffu,
                      mbar_wait(&bars->k_full[it % C::kKStages], (it / C::kKStages) & 1, w, kSiteQKs));
      if (!ok) break;
      const int* slot = bars->step[it & 3];
      if (slot[0] < 0) break;
      const int kj = slot[1], kn = slot[2], kkind = slot[3];
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->s_full[it & 1], (it >> 1) & 1, w, kSiteQS));
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars->dp_full, it & 1, w, kSiteQDp));
      if (!ok) break;
      tc_fence_after();
      const uint32_t cS = col_sq(it & 1);
      if (kkind != kFull) {
        // rewrite the scores this query does not see to -inf (P = 0 there)
        const int k0 = kn * kBN;
        int lim = min(127, g.L - k0 - 1);  // keys at or past L are padding
        if (aligned && g.causal) lim = min(lim, pos_q - token_pos<kSub>(g, kj, k0));
        int first = 0;  // first visible column (documents: keys from the row's document start)
        if constexpr (kMask) {
          const int kpos0 = token_pos<kSub>(g, kj, k0);  // tiles are contiguous under a mask
          if (doc_hi != INT_MAX) lim = min(lim, doc_hi - 1 - kpos0);
          first = max(0, doc_lo - kpos0);
        }
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
          const int c0 = cbase + half * 32;
          uint32_t vis;  // bit c: key column c0 + c is visible
          if (aligned) {
            const int nb = min(max(lim - c0 + 1, 0), 32);
            vis = nb >= 32 ? 0xFFFFFFFFu : ((1u << nb) - 1u);
            if constexpr (kMask) {
              const int nlo = min(max(first - c0, 0), 32);  // leading invisible columns
              vis &= nlo >= 32 ? 0u : (0xFFFFFFFFu << nlo);
            }
          } else {
            vis = 0u;
            for (int c = 0; c < 32; ++c) {
              const int tau = k0 + c0 + c;
              if (tau < g.L && (!g.causal || token_pos<kSub>(g, kj, tau) <= pos_q)) vis |= 1u << c;
            }
          }
          uint32_t r[32];
          tmem_ld32(trow + cS + c0, r);
          tmem_ld_wait();
          reg_fence32(r);
#pragma unroll
          for (int c = 0; c < 32; ++c)
            if (!((vis >> c) & 1u)) r[c] = 0xFF800000u;  // -inf
          tmem_st32(trow + cS + c0, r);
        }
        tmem_st_wait();
      }
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int c0 = cbase + half * 32;
        uint32_t rs[32], rp[32];
        tmem_ld32(trow + cS + c0, rs);
        tmem_ld32(trow + kColDPq + c0, rp);
        tmem_ld_wait();
        reg_fence32(rs);
        reg_fence32(rp);
        if (half == 1) {  // every dP column of this thread has been read
          tc_fence_before();
          mbar_arrive_warp(&bars->dp_free);
        }
        uint32_t dk[16];
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          const float2 x = ffma2(make_float2(__uint_as_float(rs[c]), __uint_as_float(rs[c + 1])), sl2, nl2);
          const float2 pv = make_float2(ex2_approx(x.x), ex2_approx(x.y));  // -inf -> 0
          // dS without the softmax scale (applied to dQ at the end)
          const float2 ds = fmul2(pv, fadd2(make_float2(__uint_as_float(rp[c]), __uint_as_float(rp[c + 1])), nd2));
          dk[c >> 1] = pack_bf16x2(ds.x, ds.y);
        }
        // dS back into TMEM over the S columns this thread has read
        tmem_st16(trow + cS + cbase + half * 16, dk);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive_warp(&bars->ds_full);
    }
    // ------------------------------------------------------------ epilogue: dQ rows
    if (ok && it >= 1)
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->dq_done[(it - 1) & 1], ((it - 1) >> 1) & 1, w, kSiteQEpi));
    // adding the dQ of a query tile that saw no key changes nothing (unless this call
    // writes the bf16 result, or is a dilated pair that writes the accumulator)
    const bool noop = it == 0 && (kLocal || kSub) && a.dq == nullptr && !(kSub && a.sub.first);
    if (ok && !noop) {
      tc_fence_after();
      const bool store = tau_q < g.Lq;
      size_t qr;
      if constexpr (kSub) {  // the query's original position in [B][S][Hq]
        const int pb = prob / a.sub.n_seg, ps = prob % a.sub.n_seg;
        qr = (static_cast<size_t>(pb) * a.sub.S + static_cast<size_t>(ps) * a.sub.w + a.sub.off +
              static_cast<size_t>(store ? tau_q : 0) * a.sub.r) * a.sub.Hq + (a.sub.out_h0 + h * a.sub.out_hstep);
      } else {
        qr = (static_cast<size_t>(rank * g.B + b) * g.L + (store ? tau_q : 0)) * g.Hq_l + h;
      }
#pragma unroll
      for (int c0 = wg * (D / 2); c0 < (wg + 1) * (D / 2); c0 += 32) {
        uint32_t o[32];
        if (it >= 1) {
          tmem_ld32(trow + kColDQ + c0, o);
          tmem_ld_wait();
          reg_fence32(o);
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = 0u;
        }
        if (store && (kLocal || kSub)) {
          // add this step's dQ to the fp32 accumulator; on the last step (a bf16
          // output given) write the sum as bf16 instead
          const float4* acc = reinterpret_cast<const float4*>(a.dq_acc + qr * D + c0);
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            // (a dilated pair with r = 1 run first writes the accumulator: nothing to read)
            const float4 ov = (kSub && a.sub.first) ? make_float4(0.f, 0.f, 0.f, 0.f) : acc[q];
            o[q * 4 + 0] = __float_as_uint(ov.x + __uint_as_float(o[q * 4 + 0]) * g.scale);
            o[q * 4 + 1] = __float_as_uint(ov.y + __uint_as_float(o[q * 4 + 1]) * g.scale);
            o[q * 4 + 2] = __float_as_uint(ov.z + __uint_as_float(o[q * 4 + 2]) * g.scale);
            o[q * 4 + 3] = __float_as_uint(ov.w + __uint_as_float(o[q * 4 + 3]) * g.scale);
          }
          if (a.dq == nullptr) {
            float4* dst = reinterpret_cast<float4*>(a.dq_acc + qr * D + c0);
#pragma unroll
            for (int q = 0; q < 8; ++q)
              dst[q] = make_float4(__uint_as_float(o[q * 4]), __uint_as_float(o[q * 4 + 1]),
                                   __uint_as_float(o[q * 4 + 2]), __uint_as_float(o[q * 4 + 3]));
          } else {
            uint4* dst = reinterpret_cast<uint4*>(a.dq + qr * D + c0);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint4 v;
              v.x = pack_bf16x2(__uint_as_float(o[q * 8 + 0]), __uint_as_float(o[q * 8 + 1]));
              v.y = pack_bf16x2(__uint_as_float(o[q * 8 + 2]), __uint_as_float(o[q * 8 + 3]));
              v.z = pack_bf16x2(__uint_as_float(o[q * 8 + 4]), __uint_as_float(o[q * 8 + 5]));
              v.w = pack_bf16x2(__uint_as_float(o[q * 8 + 6]), __uint_as_float(o[q * 8 + 7]));
              dst[q] = v;
            }
          }
        } else if (store) {
          uint4* dst = reinterpret_cast<uint4*>(a.dq + qr * D + c0);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(o[q * 8 + 0]) * g.scale, __uint_as_float(o[q * 8 + 1]) * g.scale);
            v.y = pack_bf16x2(__uint_as_float(o[q * 8 + 2]) * g.scale, __uint_as_float(o[q * 8 + 3]) * g.scale);
            v.z = pack_bf16x2(__uint_as_float(o[q * 8 + 4]) * g.scale, __uint_as_float(o[q * 8 + 5]) * g.scale);
            v.w = pack_bf16x2(__uint_as_float(o[q * 8 + 6]) * g.scale, __uint_as_float(o[q * 8 + 7]) * g.scale);
            dst[q] = v;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemColsDq);
  }
}

template <int D, bool kMask, int kMode>
cudaError_t launch_dq_d(const BwdLaunch& L, cudaStream_t stream) {
  constexpr bool kLocal = kMode == kModeLocal;
  constexpr bool kSub = kMode == kModeSub;
  using C = DqCfg<D>;
  static_assert(C::kSmemBytes <= 227 * 1024, "shared memory budget");
  cudaError_t e = cudaFuncSetAttribute(attn_bwd_dq_kernel<D, kMask, kMode>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  DqArgs a{};
  a.g = make_geo(L.g);
  a.g.mask = L.mask;
  a.nlse2 = L.lse2;
  a.ndelta = L.delta;
  a.Lp = L.Lp;
  a.dq = static_cast<__nv_bfloat16*>(L.dq);
  a.dq_acc = L.dq_acc;
  a.loc_i = L.loc_i;
  a.loc_u = L.loc_u;
  a.loc_t = L.loc_t;
  a.status = L.status;
  a.wait_ns = L.wait_ns;
  a.sub = L.sub;
  if (kSub) {  // one-rank geometry of every problem (see the forward's sub-problem mode)
    a.g.P_u = a.g.P_r = a.g.P = a.g.n_ranks = 1;
    a.g.L = L.sub.L;
    a.g.c = kBN;
    a.g.Lq = L.sub.Lq;
    a.g.q_off = L.sub.q_off;
    a.g.n_qtiles = (L.sub.Lq + kBM - 1) / kBM;
    a.g.n_ktiles = (L.sub.L + kBN - 1) / kBN;
  }
  const long long blocks = kSub     ? static_cast<long long>(a.g.n_qtiles) * L.sub.n_heads * L.sub.n_prob
                           : kLocal ? static_cast<long long>(a.g.n_qtiles) * a.g.B * a.g.Hq_l
                                    : static_cast<long long>(a.g.n_qtiles) * a.g.P_r * a.g.P_u * a.g.B * a.g.Hq_l;
  if (blocks <= 0) return cudaSuccess;
  if (blocks > 0x7FFFFFFFLL) return cudaErrorInvalidConfiguration;
  attn_bwd_dq_kernel<D, kMask, kMode><<<static_cast<unsigned>(blocks), kThreadsDq, C::kSmemBytes, stream>>>(
      L.tm_q, L.tm_k, L.tm_v, L.tm_do, a);
  note_launch();
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_bwd_dq(const BwdLaunch& L, cudaStream_t stream) {
  const bool masked = L.mask.bm != nullptr || L.mask.cu != nullptr;
  if (masked && (L.local || L.sub.active)) return cudaErrorInvalidValue;
  if (L.sub.active) {
    if (L.g.D == 128) return launch_dq_d<128, false, kModeSub>(L, stream);
    if (L.g.D == 64) return launch_dq_d<64, false, kModeSub>(L, stream);
    return cudaErrorInvalidValue;
  }
  if (L.local) {
    if (L.g.D == 128) return launch_dq_d<128, false, kModeLocal>(L, stream);
    if (L.g.D == 64) return launch_dq_d<64, false, kModeLocal>(L, stream);
    return cudaErrorInvalidValue;
  }
  if (masked) {
    if (L.g.D == 128) return launch_dq_d<128, true, kModeUsp>(L, stream);
    if (L.g.D == 64) return launch_dq_d<64, true, kModeUsp>(L, stream);
    return cudaErrorInvalidValue;
  }
  if (L.g.D == 128) return launch_dq_d<128, false, kModeUsp>(L, stream);
  if (L.g.D == 64) return launch_dq_d<64, false, kModeUsp>(L, stream);
  return cudaErrorInvalidValue;
}

}  // namespace usp
