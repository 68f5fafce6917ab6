// usp_attn_fwd.cu -- forward of exact softmax attention for every virtual rank
// of the USP mesh, block by block over the ring's KV chunks, on sm_100a.
//
// What it computes: for each ring rank i, Ulysses rank u, batch b and local
// query head h, the exact attention of every query row over the keys of every
// ring step t (owner j = (i - t) mod P_r), i.e. Ring Attention ("Boosting Spec
// Eagle", "The Solution") evaluated blockwise (Blockwise Parallel Transformer;
// LongNet slides, "Results": FlashAttention-style exact attention). The partial
// results of the ring steps are merged by log-sum-exp; in fused mode that merge
// happens online inside the kernel, in stepwise mode the kernel runs one ring
// step and writes the fp32 partial (O_t, LSE_t) for usp_lse_merge.
//
// CTA = two consecutive 128-row query tiles of one (rank, batch, head) that
// share every K/V tile (352 threads):
//   warp 0      TMA producer of Q0, Q1 (once) and of the K tiles (3 stages); it
//               walks the key tiles and publishes one descriptor per tile.
//   warp 10     TMA producer of the V tiles of the same walk (2 stages at D=128).
//               A K stage is released when both S of its tile have completed, a
//               V stage when both PV have: K runs ahead of the S it feeds instead
//               of waiting behind the previous tile's PV.
//   warp 1      TMEM allocator and UMMA issuer (one thread), per key tile and
//               query tile t = 0, 1 in turn:
//                 O_t += P_t V    (M=128 N=D; A = P_t read from TMEM; in two
//                                 halves of 64 keys, the first as soon as
//                                 softmax t has written that half of P_t)
//                 S_t  = Q_t K^T  of the next key tile (M=128 N=128, fp32 in TMEM;
//                                 it overwrites P_t, so it waits for that PV)
//               so the tensor core runs tile 1's PV and S while softmax 0 works
//               and the other way round. Before each S_t it hands that tile's
//               descriptor to softmax t (desc_full[t]).
//   warps 2..5  softmax of tile 0, warps 6..9 softmax of tile 1: thread = query
//               row = TMEM lane. tcgen05.ld of S, mask by original positions,
//               online max/sum in the exp2 domain with lazy rescaling of O (only
//               when the row max grows by more than 2^8), P written back as bf16
//               into the first 64 columns of S, and finally O normalised and
//               written as bf16 (LSE fp32).
// TMEM columns: S_t / P_t at 128 t, O_t at 256 + 128 t.
//
// Synchronisation is by mbarriers only; every wait is bounded (usp_ptx.cuh).
#include <math.h>

#include "usp_attn_common.cuh"
#include "usp_internal.h"
#include "usp_ptx.cuh"

namespace usp {
namespace {

constexpr int kThreadsFwd = 352;
constexpr int kWarpV = 10;  // V producer
enum : int { kModeUsp = 0, kModeSub = 1, kModeLocal = 2 };
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThresh = 8.0f;  // log2 units: rescale O only if the max grows by > 256x

__host__ __device__ constexpr uint32_t col_s(int t) { return 128u * t; }
__host__ __device__ constexpr uint32_t col_o(int t) { return 256u + 128u * t; }

template <int D>
struct FwdCfg {
  static constexpr int kPanels = D / 64;          // 128-byte (64 x bf16) swizzle panels along D
  static constexpr int kPanelBytes = 128 * 128;   // 128 rows x 128 bytes
  static constexpr int kTileBytes = kPanels * kPanelBytes;
  static constexpr int kKSt = 3;                  // K stages
  static constexpr int kVSt = D == 128 ? 2 : 3;   // V stages
  static constexpr int kOffQ = 0;                 // two query tiles
  static constexpr int kOffK = kOffQ + 2 * kTileBytes;
  static constexpr int kOffV = kOffK + kKSt * kTileBytes;
  static constexpr int kOffBar = kOffV + kVSt * kTileBytes;
  static constexpr int kSmemBytes = kOffBar + 320 + 1024;
};

struct FwdArgs {
  Geo g;
  __nv_bfloat16* out;
  float* lse;
  float* o_part;
  float* lse_part;
  int step;  // -1 fused, else the ring step
  int* status;
  unsigned long long wait_ns;
  FwdSub sub;  // sub-problem mode (kSub): see usp_internal.h
  int loc_i, loc_u;  // local mode: the one rank (ring i, Ulysses u) this launch computes
  int fold;          // step >= 0: fold into o_part / lse_part instead of writing them
};

struct FwdBars {
  uint64_t q_full;
  uint64_t k_full[3], v_full[3], k_empty[3], v_empty[3];
  uint64_t s_full[2], p_full[2], pv_done[2], desc_full[2];
  uint64_t p_half[2];  // P_t of the tile's first 64 keys is in TMEM (the first half of PV_t may start)
  uint64_t drain;
  // Key-tile descriptors published by the producer with k_full of that tile:
  // {1, or -1 = no more tiles; ring rank j of the key owner; key tile n;
  //  kind for query tile 0 | kind for query tile 1 << 4}.
  int step[4][4];
  // The descriptor of the tile whose S the MMA warp issues next for query tile
  // t, handed to that tile's softmax warps with desc_full[t].
  int sdesc[2][4];
  uint32_t tmem_base;
  int abort_flag;
};

// Wait-site codes recorded in the status word: 0x100 | role << 4 | which.
enum : int {
  kSiteQ = 0x101, kSiteKEmpty = 0x102, kSiteVEmpty = 0x103, kSiteK = 0x111, kSitePvDone = 0x112, kSiteP = 0x113,
  kSiteV = 0x114, kSiteS = 0x121, kSiteO = 0x122, kSiteDesc = 0x123
};

// The pair of consecutive query tiles (i, m, m+1) handled by CTA-order index o
// (increasing original position of the pair).
__device__ __forceinline__ void pair_in_position_order(const Geo& g, int o, int& i, int& m) {
  const int tpc = g.c / kBM;
  if (g.c % kBM == 0 && (tpc & 1) == 0) {
    tile_in_position_order(g, 2 * o, i, m);  // even tile index inside a chunk of an even number of tiles
  } else {
    const int np = (g.n_qtiles + 1) / 2;
    i = o / np;
    m = 2 * (o % np);
  }
}

// kMode: kModeUsp -- every virtual rank of the mesh, Q/K/V of all ranks in one
// head-sharded tensor; kModeSub -- independent one-rank problems (dilated
// attention); kModeLocal -- ONE rank (i, u) of a real multi-GPU mesh: its own Q
// ([B][L][Hq/P_u][D]) against the one KV block it holds at ring step `step`
// (owner j = (i - step) mod P_r, [B][L][Hkv/P_u][D]), positions as in the mesh.
template <int D, int kMode, bool kMask>
__global__ void __launch_bounds__(kThreadsFwd, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const FwdArgs a) {
  constexpr bool kSub = kMode == kModeSub;
  constexpr bool kLocal = kMode == kModeLocal;
  using C = FwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  FwdBars* bars = reinterpret_cast<FwdBars*>(smem + C::kOffBar);
  static_assert(sizeof(FwdBars) <= 320, "barrier block");
  uint8_t* sQ = smem + C::kOffQ;
  uint8_t* sK = smem + C::kOffK;
  uint8_t* sV = smem + C::kOffV;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Geo& g = a.g;  // in the sub-problem mode: the one-rank geometry of every problem
  int h, u, b, i, m, qc4;
  if constexpr (kSub) {
    // work item: (problem, head, pair of query tiles), the pairs of a (problem,
    // head) heaviest first
    const int np = (g.n_qtiles + 1) / 2;
    int wi = blockIdx.x;
    const int order = np - 1 - wi % np;
    wi /= np;
    h = a.sub.h0 + (wi % a.sub.n_heads) * a.sub.h_step;
    qc4 = wi / a.sub.n_heads;  // the problem
    u = b = i = 0;
    m = 2 * order;
  } else if constexpr (kLocal) {
    // work item: (b, head, pair of query tiles) of the one rank, heaviest first
    const int np = (g.n_qtiles + 1) / 2;
    int wi = blockIdx.x;
    const int order = np - 1 - wi % np;
    wi /= np;
    h = wi % g.Hq_l;
    b = wi / g.Hq_l;
    i = a.loc_i;
    u = a.loc_u;
    m = 2 * order;
    qc4 = 0;
  } else {
    // Work item: CTAs of one (b, Ulysses rank, head) run together so that its K/V
    // stay in L2; inside it, query-tile pairs in decreasing original position
    // (the causally heaviest first).
    const int np = (g.n_qtiles + 1) / 2;
    const int n_pairs = g.P_r * np;
    int wi = blockIdx.x;
    const int order = n_pairs - 1 - wi % n_pairs;
    wi /= n_pairs;
    h = wi % g.Hq_l;
    wi /= g.Hq_l;
    u = wi % g.P_u;
    b = wi / g.P_u;
    pair_in_position_order(g, order, i, m);
    qc4 = 0;
  }
  const int rank = (kSub || kLocal) ? 0 : i * g.P_u + u;  // local buffers hold one rank
  const int kvh = h / g.G;
  const int q0 = m * kBM;
  const int t_begin = a.step < 0 ? 0 : a.step;
  const int t_end = a.step < 0 ? g.P_r : a.step + 1;

  if (threadIdx.x == 0) {
    // A CTA that starts after another one gave up does no work at all.
    bars->abort_flag = *reinterpret_cast<volatile int*>(a.status) != 0;
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < 3; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bars->s_full[t], 1);
      mbar_init(&bars->p_full[t], 4);  // one arrival per softmax warp
      mbar_init(&bars->p_half[t], 4);
      mbar_init(&bars->pv_done[t], 1);
      mbar_init(&bars->desc_full[t], 1);
    }
    mbar_init(&bars->drain, 1);
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(&bars->tmem_base, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const WaitCtl w{&bars->abort_flag, a.status, a.wait_ns};
  const bool skip = bars->abort_flag != 0;

  if (skip) {
    // nothing issued, nothing to drain
  } else if (warp == 0 || warp == kWarpV) {
    // ------------------------------------------------------------ TMA producers
    // Warp 0 loads Q0, Q1 and the K tiles and publishes one descriptor per key
    // tile; warp kWarpV loads the V tiles of the same walk. K and V have their
    // own rings: a K stage is released as soon as both S of its tile have
    // completed, a V stage only after both PV, so K runs up to kKSt tiles ahead
    // of the S it feeds. The whole warp walks the tiles (the same values in
    // every lane); one elected lane issues each copy and barrier operation.
    {
      const bool kside = warp == 0;
      int qmin0, qmax0, qmin1, qmax1;
      qpos_range<kSub>(g, i, q0, q0 + kBM, qmin0, qmax0);
      qpos_range<kSub>(g, i, q0 + kBM, q0 + 2 * kBM, qmin1, qmax1);
      const int qmin = min(qmin0, qmin1), qmax = max(qmax0, qmax1);
      // masked variant: both query tiles' kinds narrowed by the block / document
      // masks; a key tile is walked when either query tile attends it
      const int hg = u * g.Hq_l + h;
      auto kinds_of = [&](int j, int n) {
        int k0c = classify_tile<kSub>(g, qmin0, qmax0, j, n), k1c = classify_tile<kSub>(g, qmin1, qmax1, j, n);
        int kmin, kmax;
        pos_range<kSub>(g, j, n * kBN, n * kBN + kBN, kmin, kmax);
        k0c = mask_tile(g.mask, k0c, b, hg, qmin0, qmax0, kmin, kmax);
        k1c = mask_tile(g.mask, k1c, b, hg, qmin1, qmax1, kmin, kmax);
        return k0c | (k1c << 4);
      };
      KvWalk kw;
      if constexpr (kMask)
        kw = kv_walk_begin_by(g, i, t_begin, t_end, kinds_of);
      else
        kw = kv_walk_begin<kSub>(g, i, qmin, qmax, t_begin, t_end);
      int issued = 0;
      const bool any = kw.valid;
      const int n_st = kside ? C::kKSt : C::kVSt;
      uint64_t* full = kside ? bars->k_full : bars->v_full;
      uint64_t* empty = kside ? bars->k_empty : bars->v_empty;
      const CUtensorMap* tm = kside ? &tm_k : &tm_v;
      uint8_t* sbuf = kside ? sK : sV;
      if (any) {
        if (lane == 0) {
          if (kside) tma_prefetch_desc(&tm_q);
          tma_prefetch_desc(tm);
        }
        __syncwarp();
        if (kside) {
          mbar_expect_tx_w(&bars->q_full, 2 * C::kTileBytes);
          for (int t = 0; t < 2; ++t)
            for (int p = 0; p < C::kPanels; ++p)
              tma_load_4d_w(&tm_q, &bars->q_full, sQ + t * C::kTileBytes + p * C::kPanelBytes, p * 64, h,
                            q0 + t * kBM, kSub ? qc4 : rank * g.B + b);
        }
      }
      while (true) {
        const int s = issued % n_st;
        if (!kside && !kw.valid) break;
        if (issued >= n_st &&
            !mbar_wait_w(&empty[s], ((issued / n_st) - 1) & 1, w, kside ? kSiteKEmpty : kSiteVEmpty))
          break;
        if (kside) {
          int* slot = bars->step[issued & 3];
          if (!kw.valid) {  // publish the end of the walk on this stage's barrier
            if (lane == 0) slot[0] = -1;
            __syncwarp();
            mbar_arrive_w(&full[s]);
            break;
          }
          const int kinds = kMask ? kw.kind
                                  : classify_tile<kSub>(g, qmin0, qmax0, kw.j, kw.n) |
                                        (classify_tile<kSub>(g, qmin1, qmax1, kw.j, kw.n) << 4);
          if (lane == 0) {
            slot[0] = 1;
            slot[1] = kw.j;
            slot[2] = kw.n;
            slot[3] = kinds;
          }
          __syncwarp();
        }
        const int krb = kSub ? qc4 : kLocal ? b : (kw.j * g.P_u + u) * g.B + b;
        mbar_expect_tx_w(&full[s], C::kTileBytes);
        for (int p = 0; p < C::kPanels; ++p)
          tma_load_4d_w(tm, &full[s], sbuf + s * C::kTileBytes + p * C::kPanelBytes, p * 64, kvh, kw.n * kBN, krb);
        ++issued;
        if constexpr (kMask)
          kv_walk_next_by(g, i, t_end, kw, kinds_of);
        else
          kv_walk_next<kSub>(g, i, qmin, qmax, t_end, kw);
      }
      if (*reinterpret_cast<volatile int*>(&bars->abort_flag)) {
        // Let every copy this warp started land before the CTA exits.
        if (any && kside) mbar_wait_drain(&bars->q_full, 0, a.wait_ns);
        for (int it = issued - n_st < 0 ? 0 : issued - n_st; it < issued; ++it)
          mbar_wait_drain(&full[it % n_st], (it / n_st) & 1, a.wait_ns);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ UMMA issuer
    // The whole warp runs this loop; one elected lane issues each UMMA/commit.
    {
      constexpr uint32_t kIdescQK = idesc_bf16_f32(kBM, kBN, 0, 0);
      constexpr uint32_t kIdescPV = idesc_bf16_f32(kBM, D, 0, 1);
      // descriptors of the tile bases; the start address is the low field, so a
      // byte offset inside shared memory adds (offset >> 4)
      const uint64_t dQ0 = sdesc_sw128(smem_addr(sQ), 16, 1024);
      const uint64_t dK0 = sdesc_sw128(smem_addr(sK), 16, 1024);
      const uint64_t dV0 = sdesc_sw128(smem_addr(sV), C::kPanelBytes, 1024);
      auto issue_s = [&](int t, int ks) {  // S_t = Q_t K^T, K from stage ks
        const uint64_t qd = dQ0 + ((t * C::kTileBytes) >> 4), kd = dK0 + ((ks * C::kTileBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * C::kPanelBytes + (kk & 3) * 32) >> 4;
          umma_bf16_w(tmem + col_s(t), qd + off, kd + off, kIdescQK, kk > 0 ? 1u : 0u);
        }
        umma_commit_w(&bars->s_full[t]);
      };
      // Hands the descriptor of key-tile slot `slot` (or the end of the walk) to
      // the softmax warps of query tile t.
      auto publish = [&](int t, const int* slot) {
        if (lane == 0) {
          int* sd = bars->sdesc[t];
          sd[0] = slot ? slot[0] : -1;
          if (slot) {
            sd[1] = slot[1];
            sd[2] = slot[2];
            sd[3] = slot[3];
          }
        }
        __syncwarp();
        mbar_arrive_w(&bars->desc_full[t]);
      };
      bool ok = true, issued_any = false;
      if constexpr (kMask) {
        // A query tile whose kind for a key tile is skip gets neither S nor PV of
        // it, and its softmax warps never see the tile (the walk only holds tiles
        // that at least one of the two query tiles attends). Each query tile counts
        // its own products: npv[t] PV issued; the parities of its barriers follow.
        auto attends = [](const int* slot, int t) { return ((slot[3] >> (4 * t)) & 15) != kSkip; };
        int npv[2] = {0, 0};
        bool pv_wait[2] = {false, false};  // a PV_t issued whose completion has not been waited for
        ok = mbar_wait_w(&bars->k_full[0], 0, w, kSiteK);
        const bool have = ok && bars->step[0][0] >= 0;
        if (ok && !have) {
          publish(0, nullptr);
          publish(1, nullptr);
        }
        if (have) ok = mbar_wait_w(&bars->q_full, 0, w, kSiteQ);
        if (ok && have) {
          tc_fence_after();
          const int* sl = bars->step[0];
          for (int t = 0; t < 2; ++t) {
            if (!attends(sl, t)) continue;
            publish(t, sl);
            issue_s(t, 0);
          }
          umma_commit_w(&bars->k_empty[0]);
          issued_any = true;
        }
        // Per key tile `it`, per query tile t in turn: O_t += P_t V, then S_t of
        // tile it+1 (which overwrites P_t, so it waits for that PV to land). The
        // softmax of one query tile thus overlaps the other tile's PV and S.
        for (int it = 0; ok && have; ++it) {
          const int s = it % C::kVSt;
          const int s1 = (it + 1) % C::kKSt;
          const int* cur = bars->step[it & 3];
          const bool att1 = attends(cur, 1);
          if (!mbar_wait_w(&bars->v_full[s], (it / C::kVSt) & 1, w, kSiteV)) { ok = false; break; }
          const uint64_t vd = dV0 + ((s * C::kTileBytes) >> 4);
          bool next = false;
          const int* nxt = nullptr;
          for (int t = 0; t < 2 && ok; ++t) {
            if (attends(cur, t)) {
              // PV in two halves of 64 keys: the first as soon as their P is in TMEM
              if (!mbar_wait_w(&bars->p_half[t], npv[t] & 1, w, kSiteP)) { ok = false; break; }
              tc_fence_after();
  #pragma unroll
              for (int kk = 0; kk < kBN / 32; ++kk)
                umma_bf16_tmem_a_w(tmem + col_o(t), tmem + col_s(t) + kk * 8, vd + ((kk * 16 * 128) >> 4), kIdescPV,
                                   (npv[t] > 0 || kk > 0) ? 1u : 0u);
              if (!mbar_wait_w(&bars->p_full[t], npv[t] & 1, w, kSiteP)) { ok = false; break; }
              tc_fence_after();
  #pragma unroll
              for (int kk = kBN / 32; kk < kBN / 16; ++kk)
                umma_bf16_tmem_a_w(tmem + col_o(t), tmem + col_s(t) + kk * 8, vd + ((kk * 16 * 128) >> 4), kIdescPV, 1u);
              umma_commit_w(&bars->pv_done[t]);
              ++npv[t];
              pv_wait[t] = true;
              if (t == 1 || !att1) umma_commit_w(&bars->v_empty[s]);  // the tile's last PV
            }
            if (t == 0) {
              if (!mbar_wait_w(&bars->k_full[s1], ((it + 1) / C::kKSt) & 1, w, kSiteK)) { ok = false; break; }
              nxt = bars->step[(it + 1) & 3];
              next = nxt[0] >= 0;
            }
            if (next) {
              if (attends(nxt, t)) {
                if (pv_wait[t]) {
                  if (!mbar_wait_w(&bars->pv_done[t], (npv[t] - 1) & 1, w, kSitePvDone)) { ok = false; break; }
                  pv_wait[t] = false;
                }
                tc_fence_after();
                publish(t, nxt);
                issue_s(t, s1);
              }
              if (t == 1) umma_commit_w(&bars->k_empty[s1]);  // after the tile's S
            } else {
              publish(t, nullptr);
            }
          }
          if (!ok || !next) break;
        }
      } else {
        // (no skip tiles to speak of without a mask: the plain loop, which
        // measured faster than the counting one above on dense causal work)
        ok = mbar_wait_w(&bars->k_full[0], 0, w, kSiteK);
        const bool have = ok && bars->step[0][0] >= 0;
        if (ok && !have) {
          publish(0, nullptr);
          publish(1, nullptr);
        }
        if (have) ok = mbar_wait_w(&bars->q_full, 0, w, kSiteQ);
        if (ok && have) {
          tc_fence_after();
          publish(0, bars->step[0]);
          publish(1, bars->step[0]);
          issue_s(0, 0);
          issue_s(1, 0);
          umma_commit_w(&bars->k_empty[0]);
          issued_any = true;
        }
        // Per key tile `it`, per query tile t in turn: O_t += P_t V, then S_t of
        // tile it+1 (which overwrites P_t, so it waits for that PV to land). The
        // softmax of one query tile thus overlaps the other tile's PV and S.
        for (int it = 0; ok && have; ++it) {
          const int s = it % C::kVSt;
          const int s1 = (it + 1) % C::kKSt;
          if (!mbar_wait_w(&bars->v_full[s], (it / C::kVSt) & 1, w, kSiteV)) { ok = false; break; }
          const uint64_t vd = dV0 + ((s * C::kTileBytes) >> 4);
          bool next = false;
          for (int t = 0; t < 2 && ok; ++t) {
            // PV in two halves of 64 keys: the first as soon as their P is in TMEM
            if (!mbar_wait_w(&bars->p_half[t], it & 1, w, kSiteP)) { ok = false; break; }
            tc_fence_after();
  #pragma unroll
            for (int kk = 0; kk < kBN / 32; ++kk)
              umma_bf16_tmem_a_w(tmem + col_o(t), tmem + col_s(t) + kk * 8, vd + ((kk * 16 * 128) >> 4), kIdescPV,
                                 (it > 0 || kk > 0) ? 1u : 0u);
            if (!mbar_wait_w(&bars->p_full[t], it & 1, w, kSiteP)) { ok = false; break; }
            tc_fence_after();
  #pragma unroll
            for (int kk = kBN / 32; kk < kBN / 16; ++kk)
              umma_bf16_tmem_a_w(tmem + col_o(t), tmem + col_s(t) + kk * 8, vd + ((kk * 16 * 128) >> 4), kIdescPV, 1u);
            umma_commit_w(&bars->pv_done[t]);
            if (t == 1) umma_commit_w(&bars->v_empty[s]);
            if (t == 0) {
              if (!mbar_wait_w(&bars->k_full[s1], ((it + 1) / C::kKSt) & 1, w, kSiteK)) { ok = false; break; }
              next = bars->step[(it + 1) & 3][0] >= 0;
            }
            if (next) {
              if (!mbar_wait_w(&bars->pv_done[t], it & 1, w, kSitePvDone)) { ok = false; break; }
              tc_fence_after();
              publish(t, bars->step[(it + 1) & 3]);
              issue_s(t, s1);
              if (t == 1) umma_commit_w(&bars->k_empty[s1]);
            } else {
              publish(t, nullptr);
            }
          }
          if (!ok || !next) break;
        }
      }
      if (!ok && issued_any) {
        umma_commit_w(&bars->drain);
        mbar_wait_drain(&bars->drain, 0, a.wait_ns);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax warpgroups
    const int t = (warp - 2) >> 2;  // query tile of this warpgroup
    const int wq = warp & 3;        // TMEM lane quarter
    const int row = wq * 32 + lane;
    const uint32_t trow = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const uint32_t cS = col_s(t), cO = col_o(t);
    const int tau_q = q0 + t * kBM + row;
    const int pos_q = tau_q < g.Lq ? qtoken_pos<kSub>(g, i, tau_q) : INT_MAX;
    const bool aligned = (g.c % kBN) == 0;
    int doc_lo = 0, doc_hi = INT_MAX;  // the row's document [lo, hi) (masked variant)
    if constexpr (kMask) doc_span(g.mask, pos_q, doc_lo, doc_hi);
    // l_run: sum of the fp32 weights (for LSE); lb_run: sum of the bf16-rounded
    // weights the PV UMMA consumes (normalises O, so O stays a convex combination
    // of V rows even when one key dominates).
    float m_use = -INFINITY, l_run = 0.f, lb_run = 0.f;
    int it = 0;
    bool ok = true;
    for (;; ++it) {
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->desc_full[t], it & 1, w, kSiteDesc));
      if (!ok) break;
      const int* slot = bars->sdesc[t];
      if (slot[0] < 0) break;
      const int kj = slot[1], kn = slot[2], kkind = (slot[3] >> (4 * t)) & 15;
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->s_full[t], it & 1, w, kSiteS));
      if (!ok) break;
      tc_fence_after();
      // Tiles that are not wholly visible: rewrite the invisible scores of this
      // row to -inf in TMEM first, so the two passes below carry no masking.
      if (kkind != kFull) {
        const int k0 = kn * kBN;
        int lim = kkind == kSkip ? -1 : min(127, g.L - k0 - 1);  // keys at or past L are padding
        if (kkind == kMasked && aligned && g.causal) lim = min(lim, pos_q - token_pos<kSub>(g, kj, k0));
        int first = 0;  // first visible column (documents: keys from the row's document start)
        if constexpr (kMask) {
          if (kkind == kMasked) {
            const int kpos0 = token_pos<kSub>(g, kj, k0);  // tiles are contiguous under a mask
            lim = min(lim, doc_hi == INT_MAX ? 127 : doc_hi - 1 - kpos0);
            first = max(0, doc_lo - kpos0);
          }
        }
        const bool per_key = kkind == kMasked && !aligned;  // chunks shorter than a tile
#pragma unroll 1
        for (int c0 = 0; c0 < 128; c0 += 32) {
          uint32_t vis;  // bit c: column c0 + c is visible
          if (!per_key) {
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
      // The whole S row in registers: one round trip to TMEM.
      uint32_t r0[32], r1[32], r2[32], r3[32];
      tmem_ld32(trow + cS + 0, r0);
      tmem_ld32(trow + cS + 32, r1);
      tmem_ld32(trow + cS + 64, r2);
      tmem_ld32(trow + cS + 96, r3);
      tmem_ld_wait();
      reg_fence32(r0);
      reg_fence32(r1);
      reg_fence32(r2);
      reg_fence32(r3);
      // row max with 8 independent partial maxima (short dependency chains)
      float pm[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) pm[q] = fmax3(__uint_as_float(r0[q]), __uint_as_float(r1[q]), __uint_as_float(r2[q]));
#pragma unroll
      for (int c = 8; c < 32; c += 8) {
#pragma unroll
        for (int q = 0; q < 8; ++q) pm[q] = fmax3(pm[q], __uint_as_float(r0[c + q]), __uint_as_float(r1[c + q]));
#pragma unroll
        for (int q = 0; q < 8; ++q) pm[q] = fmax3(pm[q], __uint_as_float(r2[c + q]), __uint_as_float(r3[c + q]));
      }
#pragma unroll
      for (int q = 0; q < 8; ++q) pm[q] = fmaxf(pm[q], __uint_as_float(r3[q]));
      const float mx = fmaxf(fmax3(pm[0], pm[1], pm[2]), fmax3(pm[3], pm[4], fmax3(pm[5], pm[6], pm[7])));
      const float m_tile = mx * g.scale_log2;
      const bool bump = m_tile > m_use + kRescaleThresh;
      float alpha = 1.f;
      if (bump) {
        alpha = ex2_approx(m_use - m_tile);
        m_use = m_tile;
      }
      const float m_safe = m_use == -INFINITY ? 0.f : m_use;
      // P = exp2(S*scale*log2e - m) as bf16 into the first 64 columns of S_t, two
      // keys per column (-inf scores give 0).
      // independent packed accumulators for the fp32 and the bf16-rounded sums
      float2 acc[4], accb[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[q] = accb[q] = make_float2(0.f, 0.f);
      const float2 sl2 = make_float2(g.scale_log2, g.scale_log2);
      const float2 nm = make_float2(-m_safe, -m_safe);
      auto emit = [&](const uint32_t (&r)[32], uint32_t col) {
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          const float2 x = ffma2(make_float2(__uint_as_float(r[c]), __uint_as_float(r[c + 1])), sl2, nm);
          const float2 pv = make_float2(ex2_approx(x.x), ex2_approx(x.y));
          acc[(c >> 1) & 3] = fadd2(acc[(c >> 1) & 3], pv);
          pk[c >> 1] = pack_bf16x2(pv.x, pv.y);
          accb[(c >> 1) & 3] = add_bf16x2_f32(accb[(c >> 1) & 3], pk[c >> 1]);
        }
        tmem_st16(trow + cS + col, pk);
      };
      emit(r0, 0);
      emit(r1, 16);
      // The PV UMMA of the previous tile has completed (S_t is only issued after
      // it), so O_t can be rescaled in place -- before the first half of P is
      // handed over, since the first half of PV_t starts on it.
      if (it > 0 && __any_sync(0xffffffffu, bump)) {
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t o[32];
          tmem_ld32(trow + cO + c0, o);
          tmem_ld_wait();
          reg_fence32(o);
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
          tmem_st32(trow + cO + c0, o);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive_warp(&bars->p_half[t]);
      emit(r2, 32);
      emit(r3, 48);
      const float rs = (acc[0].x + acc[0].y) + (acc[1].x + acc[1].y) + (acc[2].x + acc[2].y) + (acc[3].x + acc[3].y);
      const float rsb =
          (accb[0].x + accb[0].y) + (accb[1].x + accb[1].y) + (accb[2].x + accb[2].y) + (accb[3].x + accb[3].y);
      l_run = l_run * alpha + rs;
      lb_run = lb_run * alpha + rsb;
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive_warp(&bars->p_full[t]);
    }
    // ------------------------------------------------------------ epilogue
    if (ok && it >= 1) ok = __all_sync(0xffffffffu, mbar_wait(&bars->pv_done[t], (it - 1) & 1, w, kSiteO));
    // folding a tile that saw no key changes nothing (its weight is 0): no read, no write
    const bool noop = it == 0 && (kSub ? !a.sub.first : (a.step >= 0 && a.fold));
    if (ok && !noop) {
      tc_fence_after();
      const bool store = tau_q < g.Lq;
      const float inv_l = lb_run > 0.f ? 1.f / lb_run : 0.f;
      const float lse_val = l_run > 0.f ? (m_use + __log2f(l_run)) * 0.6931471805599453f : -INFINITY;
      if constexpr (kSub) {
        // fold this pair's (O_k, LSE_k) into the running fp32 (O, LSE) of the row:
        // weights exp(LSE_k - LSE) and exp(LSE_old - LSE), LSE = logaddexp of both
        const int pb = qc4 / a.sub.n_seg, ps = qc4 % a.sub.n_seg;
        const size_t orow = static_cast<size_t>(pb) * a.sub.S + static_cast<size_t>(ps) * a.sub.w + a.sub.off +
                            static_cast<size_t>(store ? tau_q : 0) * a.sub.r;
        const size_t ridx = orow * a.sub.Hq + (a.sub.out_h0 + h * a.sub.out_hstep);
        float lse_old = -INFINITY;
        if (store && !a.sub.first) lse_old = a.sub.lse_run[ridx];
        const float mx = fmaxf(lse_old, lse_val);
        float w_old = 0.f, w_new = 0.f, lse_new = -INFINITY;
        if (mx != -INFINITY) {
          const float e_old = ex2_approx((lse_old - mx) * 1.4426950408889634f);
          const float e_new = ex2_approx((lse_val - mx) * 1.4426950408889634f);
          const float inv = 1.f / (e_old + e_new);
          w_old = e_old * inv;
          w_new = e_new * inv * inv_l;
          lse_new = mx + __logf(e_old + e_new);
        }
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t o[32];
          if (it >= 1) {
            tmem_ld32(trow + cO + c0, o);
            tmem_ld_wait();
            reg_fence32(o);
          } else {
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = 0u;
          }
          if (store) {
            float4* dst = reinterpret_cast<float4*>(a.sub.o_run + ridx * D + c0);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const float4 ov = a.sub.first ? make_float4(0.f, 0.f, 0.f, 0.f) : dst[q];
              dst[q] = make_float4(ov.x * w_old + __uint_as_float(o[q * 4 + 0]) * w_new,
                                   ov.y * w_old + __uint_as_float(o[q * 4 + 1]) * w_new,
                                   ov.z * w_old + __uint_as_float(o[q * 4 + 2]) * w_new,
                                   ov.w * w_old + __uint_as_float(o[q * 4 + 3]) * w_new);
            }
          }
        }
        if (store) a.sub.lse_run[ridx] = lse_new;
      } else {
      const size_t row_idx = (static_cast<size_t>(rank * g.B + b) * g.L + (store ? tau_q : 0)) * g.Hq_l + h;
      // fp32 partial of a ring step: written (weight 1/l), or folded into the
      // running partial already there by the log-sum-exp merge
      float w_old = 0.f, w_new = inv_l, lse_out = lse_val;
      if (a.step >= 0 && a.fold && store) {
        const float lse_old = a.lse_part[row_idx];
        const float mx = fmaxf(lse_old, lse_val);
        w_new = 0.f;
        lse_out = -INFINITY;
        if (mx != -INFINITY) {
          const float e_old = ex2_approx((lse_old - mx) * 1.4426950408889634f);
          const float e_new = ex2_approx((lse_val - mx) * 1.4426950408889634f);
          const float inv = 1.f / (e_old + e_new);
          w_old = e_old * inv;
          w_new = e_new * inv * inv_l;
          lse_out = mx + __logf(e_old + e_new);
        }
      }
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t o[32];
        if (it >= 1) {
          tmem_ld32(trow + cO + c0, o);
          tmem_ld_wait();
          reg_fence32(o);
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = 0u;
        }
        if (store) {
          if (a.step < 0) {
            uint4* dst = reinterpret_cast<uint4*>(a.out + row_idx * D + c0);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint4 v;
              v.x = pack_bf16x2(__uint_as_float(o[q * 8 + 0]) * inv_l, __uint_as_float(o[q * 8 + 1]) * inv_l);
              v.y = pack_bf16x2(__uint_as_float(o[q * 8 + 2]) * inv_l, __uint_as_float(o[q * 8 + 3]) * inv_l);
              v.z = pack_bf16x2(__uint_as_float(o[q * 8 + 4]) * inv_l, __uint_as_float(o[q * 8 + 5]) * inv_l);
              v.w = pack_bf16x2(__uint_as_float(o[q * 8 + 6]) * inv_l, __uint_as_float(o[q * 8 + 7]) * inv_l);
              dst[q] = v;
            }
          } else {
            float4* dst = reinterpret_cast<float4*>(a.o_part + row_idx * D + c0);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              float4 nv = make_float4(__uint_as_float(o[q * 4 + 0]) * w_new, __uint_as_float(o[q * 4 + 1]) * w_new,
                                      __uint_as_float(o[q * 4 + 2]) * w_new, __uint_as_float(o[q * 4 + 3]) * w_new);
              if (a.fold) {
                const float4 ov = dst[q];
                nv = make_float4(nv.x + ov.x * w_old, nv.y + ov.y * w_old, nv.z + ov.z * w_old, nv.w + ov.w * w_old);
              }
              dst[q] = nv;
            }
          }
        }
      }
      if (store) {
        if (a.step < 0)
          a.lse[row_idx] = lse_val;
        else
          a.lse_part[row_idx] = lse_out;
      }
      }  // USP epilogue
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D, int kMode, bool kMask>
cudaError_t launch_fwd_d(const FwdLaunch& L, cudaStream_t stream) {
  constexpr bool kSub = kMode == kModeSub;
  using C = FwdCfg<D>;
  static_assert(C::kSmemBytes <= 227 * 1024, "shared memory budget");
  cudaError_t e = cudaFuncSetAttribute(attn_fwd_kernel<D, kMode, kMask>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  FwdArgs a{};
  a.g = make_geo(L.g);
  a.out = static_cast<__nv_bfloat16*>(L.out);
  a.lse = L.lse;
  a.o_part = L.o_part;
  a.lse_part = L.lse_part;
  a.step = L.step;
  a.status = L.status;
  a.wait_ns = L.wait_ns;
  a.sub = L.sub;
  a.g.mask = L.mask;
  long long blocks;
  if (kSub) {
    // every problem: one rank, L = sub.L rows whose local index is the position
    // (contiguous, so the aligned masking path applies)
    a.g.P_u = a.g.P_r = a.g.P = a.g.n_ranks = 1;
    a.g.L = L.sub.L;
    a.g.c = kBN;
    a.g.Lq = L.sub.Lq;
    a.g.q_off = L.sub.q_off;
    a.g.n_qtiles = (L.sub.Lq + kBM - 1) / kBM;
    a.g.n_ktiles = (L.sub.L + kBN - 1) / kBN;
    blocks = static_cast<long long>((a.g.n_qtiles + 1) / 2) * L.sub.n_heads * L.sub.n_prob;
  } else if (kMode == kModeLocal) {
    a.loc_i = L.loc_i;
    a.loc_u = L.loc_u;
    a.fold = L.fold;
    blocks = static_cast<long long>((a.g.n_qtiles + 1) / 2) * a.g.B * a.g.Hq_l;
  } else {
    blocks = static_cast<long long>((a.g.n_qtiles + 1) / 2) * a.g.P_r * a.g.P_u * a.g.B * a.g.Hq_l;
  }
  if (blocks <= 0) return cudaSuccess;
  if (blocks > 0x7FFFFFFFLL) return cudaErrorInvalidConfiguration;
  attn_fwd_kernel<D, kMode, kMask><<<static_cast<unsigned>(blocks), kThreadsFwd, C::kSmemBytes, stream>>>(
      L.tm_q, L.tm_k, L.tm_v, a);
  note_launch();
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_fwd(const FwdLaunch& L, cudaStream_t stream) {
  const bool masked = L.mask.bm != nullptr || L.mask.cu != nullptr;
  if ((L.sub.active || L.local) && masked) return cudaErrorInvalidValue;  // masks: emulated mesh only
  if (L.sub.active) {
    if (L.g.D == 128) return launch_fwd_d<128, kModeSub, false>(L, stream);
    if (L.g.D == 64) return launch_fwd_d<64, kModeSub, false>(L, stream);
    return cudaErrorInvalidValue;
  }
  if (L.local) {
    if (L.g.D == 128) return launch_fwd_d<128, kModeLocal, false>(L, stream);
    if (L.g.D == 64) return launch_fwd_d<64, kModeLocal, false>(L, stream);
    return cudaErrorInvalidValue;
  }
  if (masked) {
    if (L.g.D == 128) return launch_fwd_d<128, kModeUsp, true>(L, stream);
    if (L.g.D == 64) return launch_fwd_d<64, kModeUsp, true>(L, stream);
    return cudaErrorInvalidValue;
  }
  if (L.g.D == 128) return launch_fwd_d<128, kModeUsp, false>(L, stream);
  if (L.g.D == 64) return launch_fwd_d<64, kModeUsp, false>(L, stream);
  return cudaErrorInvalidValue;
}

}  // namespace usp
