// usp_attn_common.cuh -- geometry shared by the attention kernels: original
// token positions of the zigzag / Ulysses layout and the classification of a
// (query tile, key tile) pair for the causal mask.
//
// Zigzag reading ("Boosting Spec Eagle", "Implementation Details": load
// balancing across the ring): 2P chunks of c tokens, rank r holds chunks r and
// 2P-1-r. After the Ulysses all-to-all (DeepSpeed-Ulysses summary, "Wie
// DeepSpeed-Ulysses funktioniert"), ring rank i holds, for u' = 0..P_u-1, the
// 2c tokens of rank i*P_u + u' in order: local token tau lies in local chunk
// kappa = tau / c, which is chunk (kappa odd ? 2P-1-r' : r') with r' = i*P_u + kappa/2.
#pragma once

#include <climits>

#include "usp_internal.h"

namespace usp {

constexpr int kBM = 128;  // query rows per tile (UMMA M)
constexpr int kBN = 128;  // keys per tile

// Masks beyond causality (DeepSpeed-Ulysses summary, "Hauptmerkmale" item 3:
// dense and sparse attention under the Ulysses layout): a block mask over
// 128 x 128 blocks of original positions, and packed variable-length sequences
// (documents [cu[d], cu[d+1]) of the sequence; a query sees keys of its own
// document only). With a mask every chunk is a whole number of tiles, so the
// positions of a tile are contiguous and lie in one block.
// (MaskArgs is declared in usp_internal.h: bm [B][Hq][nb][nb] with 1 = the block
// is computed; cu [n_docs + 1] document starts with cu[0] = 0, cu[n_docs] = S.)

struct Geo {
  int B, L, Hq_l, Hkv_l, G, P_u, P_r, P, c, causal, n_ranks, n_qtiles, n_ktiles;
  int Lq, q_off;     // query rows and the position of the first (L and 0 but in a query window)
  MaskArgs mask;     // read only by the masked kernel variants
  float scale_log2;  // softmax scale * log2(e)
  float scale;       // softmax scale
};

inline Geo make_geo(const AttnGeom& a) {
  Geo g{};
  g.B = a.B; g.L = a.L; g.Hq_l = a.Hq_l; g.Hkv_l = a.Hkv_l; g.G = a.G; g.P_u = a.P_u; g.P_r = a.P_r;
  g.P = a.P; g.c = a.c; g.causal = a.causal; g.n_ranks = a.n_ranks;
  g.n_qtiles = (a.L + kBM - 1) / kBM;
  g.n_ktiles = (a.L + kBN - 1) / kBN;
  g.Lq = a.L;
  g.q_off = 0;
  g.scale = 1.0f / sqrtf(static_cast<float>(a.D));
  g.scale_log2 = g.scale * 1.4426950408889634f;
  return g;
}

// Original token position of local token tau of ring rank i (tau < L). With
// kPlain (the one-rank geometry of the sub-problem mode) tau is the position.
template <bool kPlain = false>
__device__ __forceinline__ int token_pos(const Geo& g, int i, int tau) {
  if constexpr (kPlain) return tau;
  const int kappa = tau / g.c;
  const int rp = i * g.P_u + (kappa >> 1);
  const int chunk = (kappa & 1) ? (2 * g.P - 1 - rp) : rp;
  return chunk * g.c + (tau - kappa * g.c);
}

// Smallest and largest original position among local tokens [t0, t1) of ring rank i.
template <bool kPlain = false>
__device__ __forceinline__ void pos_range(const Geo& g, int i, int t0, int t1, int& pmin, int& pmax) {
  if (t1 > g.L) t1 = g.L;
  pmin = INT_MAX;
  pmax = -1;
  if (t0 >= t1) return;  // the range lies wholly in the padding past L
  if constexpr (kPlain) {
    pmin = t0;
    pmax = t1 - 1;
  } else {
    for (int kap = t0 / g.c; kap * g.c < t1; ++kap) {
      const int a = max(t0, kap * g.c);
      const int e = min(t1, (kap + 1) * g.c) - 1;
      pmin = min(pmin, token_pos(g, i, a));
      pmax = max(pmax, token_pos(g, i, e));
    }
  }
}

// Query-side forms: the same positions, except in the sub-problem mode, where
// the g.Lq query rows of a launch are a window whose positions start at g.q_off.
template <bool kPlain = false>
__device__ __forceinline__ int qtoken_pos(const Geo& g, int i, int tau) {
  if constexpr (kPlain) return g.q_off + tau;
  return token_pos(g, i, tau);
}
template <bool kPlain = false>
__device__ __forceinline__ void qpos_range(const Geo& g, int i, int t0, int t1, int& pmin, int& pmax) {
  if constexpr (kPlain) {
    if (t1 > g.Lq) t1 = g.Lq;
    pmin = INT_MAX;
    pmax = -1;
    if (t0 >= t1) return;
    pmin = g.q_off + t0;
    pmax = g.q_off + t1 - 1;
  } else {
    pos_range(g, i, t0, t1, pmin, pmax);
  }
}

// The o-th 128-token tile of the whole sequence (all ring ranks) in increasing
// original position: returns its ring rank i and local tile index n. When a
// chunk is not a whole number of tiles the plain (rank, tile) order is used.
__device__ __forceinline__ void tile_in_position_order(const Geo& g, int o, int& i, int& n) {
  if (g.c % kBN == 0) {
    const int tpc = g.c / kBN;  // tiles per chunk
    const int chunk = o / tpc, within = o % tpc;
    const bool late = chunk >= g.P;
    const int r = late ? 2 * g.P - 1 - chunk : chunk;
    i = r / g.P_u;
    n = (2 * (r % g.P_u) + (late ? 1 : 0)) * tpc + within;
  } else {
    i = o / g.n_ktiles;
    n = o % g.n_ktiles;
  }
}

enum TileKind { kSkip = 0, kFull = 1, kMasked = 2 };

// Kind of the pair (query tile with positions [qmin, qmax], key tile n of ring rank j).
template <bool kPlain = false>
__device__ __forceinline__ int classify_tile(const Geo& g, int qmin, int qmax, int j, int n) {
  const int k0 = n * kBN;
  const bool ragged = k0 + kBN > g.L;
  if (!g.causal) return ragged ? kMasked : kFull;
  int kmin, kmax;
  pos_range<kPlain>(g, j, k0, k0 + kBN, kmin, kmax);
  if (qmax < kmin) return kSkip;
  if (qmin >= kmax && !ragged) return kFull;
  return kMasked;
}

// Document of position pos: the largest d with cu[d] <= pos.
__device__ __forceinline__ int doc_of(const int* cu, int n_docs, int pos) {
  int lo = 0, hi = n_docs - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(cu + mid) <= pos) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// The causal kind of a (query tile, key tile) pair narrowed by the masks: the
// query tile holds positions [qmin, qmax] of global query head hg (batch b),
// the key tile [kmin, kmax]. Skipped when its block is off or no document
// spans both tiles; masked (per key) when the tiles touch more than one
// document. An empty query tile (qmin > qmax) is skipped.
__device__ __forceinline__ int mask_tile(const MaskArgs& mk, int kind, int b, int hg, int qmin, int qmax, int kmin,
                                         int kmax) {
  if (kind == kSkip || qmin > qmax || kmin > kmax) return kSkip;
  if (mk.bm &&
      !__ldg(mk.bm + (static_cast<size_t>(b * mk.Hq + hg) * mk.nb + qmin / kBM) * mk.nb + kmin / kBN))
    return kSkip;
  if (mk.cu) {
    const int dq0 = doc_of(mk.cu, mk.n_docs, qmin), dq1 = doc_of(mk.cu, mk.n_docs, qmax);
    const int dk0 = doc_of(mk.cu, mk.n_docs, kmin), dk1 = doc_of(mk.cu, mk.n_docs, kmax);
    if (dq1 < dk0 || dk1 < dq0) return kSkip;
    if (dq0 != dq1 || dk0 != dk1) return kMasked;
  }
  return kind;
}

// The document interval [lo, hi) holding position pos ([0, INT_MAX) without documents).
__device__ __forceinline__ void doc_span(const MaskArgs& mk, int pos, int& lo, int& hi) {
  lo = 0;
  hi = INT_MAX;
  if (mk.cu && pos != INT_MAX) {
    const int d = doc_of(mk.cu, mk.n_docs, pos);
    lo = __ldg(mk.cu + d);
    hi = __ldg(mk.cu + d + 1);
  }
}

// Enumerates, in ring order, the non-skipped key tiles a query tile of ring
// rank i attends: steps t in [t_begin, t_end), owner j = (i - t) mod P_r,
// key tiles n = 0 .. n_ktiles-1 of rank j; `cls(j, n)` gives a tile's kind
// (0 = skip). Every role of a CTA walks the same sequence.
struct KvWalk {
  int t, n, j, kind;
  bool valid;
};

template <class Cls>
__device__ __forceinline__ void kv_walk_settle_by(const Geo& g, int i, int t_end, KvWalk& w, const Cls& cls) {
  while (w.t < t_end) {
    w.j = (i - w.t + g.P_r) % g.P_r;
    while (w.n < g.n_ktiles) {
      w.kind = cls(w.j, w.n);
      if (w.kind != kSkip) {
        w.valid = true;
        return;
      }
      ++w.n;
    }
    ++w.t;
    w.n = 0;
  }
  w.valid = false;
}

template <class Cls>
__device__ __forceinline__ KvWalk kv_walk_begin_by(const Geo& g, int i, int t_begin, int t_end, const Cls& cls) {
  KvWalk w{t_begin, 0, 0, 0, false};
  kv_walk_settle_by(g, i, t_end, w, cls);
  return w;
}

template <class Cls>
__device__ __forceinline__ void kv_walk_next_by(const Geo& g, int i, int t_end, KvWalk& w, const Cls& cls) {
  ++w.n;
  kv_walk_settle_by(g, i, t_end, w, cls);
}

// The walk by the causal kind of a query tile with positions [qmin, qmax].
template <bool kPlain = false>
__device__ __forceinline__ KvWalk kv_walk_begin(const Geo& g, int i, int qmin, int qmax, int t_begin, int t_end) {
  return kv_walk_begin_by(g, i, t_begin, t_end,
                          [&](int j, int n) { return classify_tile<kPlain>(g, qmin, qmax, j, n); });
}

template <bool kPlain = false>
__device__ __forceinline__ void kv_walk_next(const Geo& g, int i, int qmin, int qmax, int t_end, KvWalk& w) {
  kv_walk_next_by(g, i, t_end, w, [&](int j, int n) { return classify_tile<kPlain>(g, qmin, qmax, j, n); });
}

}  // namespace usp
