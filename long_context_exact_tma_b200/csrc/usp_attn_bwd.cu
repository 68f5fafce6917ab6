// usp_attn_bwd.cu -- backward of the blockwise USP attention on sm_100a.
//
// What it computes (the gradient of the forward's exact attention; the pages
// give no formula, these are the derivatives of softmax attention): with P
// recomputed from the forward's final merged LSE,
//   P_ij = exp(scale q_i.k_j - LSE_i),   dP = dO V^T,   Delta_i = sum_d dO_id O_id,
//   dS = scale * P o (dP - Delta),        dQ = dS K,   dK = dS^T Q,   dV = P^T dO,
// with dK/dV summed over the q-heads of a GQA group and over every ring rank's
// queries (in the ring algorithm dK/dV travel around the ring with K/V).
//
// CTA = one 128-key tile of one kv-head of one head-sharded rank (i.e. the
// ring's KV chunk owner). It loops over the q-heads of the group, the ring
// ranks whose queries see the tile, and their 128-row query tiles:
//   warp 0      TMA: K, V once; per step Q, dO tiles and the 128 LSE/Delta values.
//   warp 1      TMEM allocator + UMMA issuer:
//                 S^T  = K Q^T        -> TMEM [0,128)      (M = keys, N = queries)
//                 dP^T = V dO^T       -> TMEM [128,256)
//                 dV  += P^T dO       -> TMEM [256,256+D)  (A = P^T from shared memory)
//                 dK  += dS^T Q       -> TMEM [384,384+D)  (A = dS^T from shared memory)
//                 dQt  = dS K         -> TMEM [0, D)       (A = dS, MN-major view of dS^T)
//   warps 2..5  thread = key row: P^T and dS^T rows from S^T/dP^T (tcgen05.ld),
//               written bf16 into 128B-swizzled shared memory; then thread =
//               query row: the dQ tile is read from TMEM and added to the fp32
//               dQ accumulator in global memory with vector atomics. At the end
//               dK and dV rows (fp32) are written out.
// Every wait is bounded (usp_ptx.cuh).
#include <math.h>

#include "usp_attn_common.cuh"
#include "usp_internal.h"
#include "usp_ptx.cuh"

namespace usp {
namespace {

constexpr int kThreadsBwd = 192;
constexpr uint32_t kTmemColsBwd = 512;
constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 384;

template <int D>
struct BwdCfg {
  static constexpr int kPanels = D / 64;
  static constexpr int kPanelBytes = 128 * 128;
  static constexpr int kTileBytes = kPanels * kPanelBytes;
  static constexpr int kStages = D == 128 ? 1 : 2;
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kTileBytes;
  static constexpr int kOffQ = 2 * kTileBytes;
  static constexpr int kOffDO = kOffQ + kStages * kTileBytes;
  static constexpr int kOffPt = kOffDO + kStages * kTileBytes;  // P^T: 128 keys x 128 queries bf16
  static constexpr int kOffDSt = kOffPt + 2 * kPanelBytes;      // dS^T
  static constexpr int kOffRow = kOffDSt + 2 * kPanelBytes;     // per stage: LSE*log2e [128], Delta [128]
  static constexpr int kOffBar = kOffRow + kStages * 1024;
  static constexpr int kSmemBytes = kOffBar + 512 + 1024;
};

struct BwdArgs {
  Geo g;
  const float* lse2;   // [n_ranks*B*Hq_l][Lp]: LSE * log2(e)
  const float* delta;  // [n_ranks*B*Hq_l][Lp]
  int Lp;
  float* dq_acc;       // fp32 [n_ranks][B][L][Hq_l][D]
  float* dk;           // fp32 [n_ranks][B][L][Hkv_l][D]
  float* dv;
  int* status;
  unsigned long long wait_ns;
};

struct BwdBars {
  uint64_t kv_full;
  uint64_t qd_full[2], qd_empty[2];
  uint64_t st_full, p_full, dq_full, dq_free, drain;
  uint32_t tmem_base;
  int abort_flag;
};

enum : int {
  kSiteBKv = 0x201, kSiteBQdEmpty = 0x202, kSiteBQd = 0x211, kSiteBDqFree = 0x212, kSiteBP = 0x213,
  kSiteBSt = 0x221, kSiteBDq = 0x222, kSiteBQdC = 0x223
};

// Query steps of one key tile: q-head hh of the group, ring rank i, query tile m.
struct QWalk {
  int hh, t, m, i, kind;
  bool valid;
};

__device__ __forceinline__ int classify_q(const Geo& g, int i, int m, int kmin, int kmax) {
  const int q0 = m * kBM;
  int qmin, qmax;
  pos_range(g, i, q0, q0 + kBM, qmin, qmax);
  if (g.causal && qmax < kmin) return kSkip;
  if (q0 + kBM > g.L) return kMasked;  // padded query columns must be masked
  if (!g.causal || qmin >= kmax) return kFull;
  return kMasked;
}

__device__ __forceinline__ void qwalk_settle(const Geo& g, int j, int kmin, int kmax, QWalk& w) {
  while (w.hh < g.G) {
    while (w.t < g.P_r) {
      w.i = (j + w.t) % g.P_r;
      while (w.m < g.n_qtiles) {
        w.kind = classify_q(g, w.i, w.m, kmin, kmax);
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
    w.t = 0;
  }
  w.valid = false;
}

__device__ __forceinline__ QWalk qwalk_begin(const Geo& g, int j, int kmin, int kmax) {
  QWalk w{0, 0, 0, 0, 0, false};
  qwalk_settle(g, j, kmin, kmax, w);
  return w;
}

__device__ __forceinline__ void qwalk_next(const Geo& g, int j, int kmin, int kmax, QWalk& w) {
  ++w.m;
  qwalk_settle(g, j, kmin, kmax, w);
}

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

template <int D>
__global__ void __launch_bounds__(kThreadsBwd, 1)
    attn_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    const BwdArgs a) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  BwdBars* bars = reinterpret_cast<BwdBars*>(smem + C::kOffBar);
  uint8_t* sK = smem + C::kOffK;
  uint8_t* sV = smem + C::kOffV;
  uint8_t* sQ = smem + C::kOffQ;
  uint8_t* sDO = smem + C::kOffDO;
  uint8_t* sPt = smem + C::kOffPt;
  uint8_t* sDSt = smem + C::kOffDSt;
  float* sRow = reinterpret_cast<float*>(smem + C::kOffRow);

  const Geo& g = a.g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  int wi = blockIdx.x;
  const int gl = wi % g.Hkv_l;
  wi /= g.Hkv_l;
  const int b = wi % g.B;
  wi /= g.B;
  const int jrank = wi % g.n_ranks;
  wi /= g.n_ranks;
  const int n = wi;
  const int j = jrank / g.P_u, u = jrank % g.P_u;
  const int k0 = n * kBN;
  int kmin, kmax;
  pos_range(g, j, k0, k0 + kBN, kmin, kmax);

  if (threadIdx.x == 0) {
    bars->abort_flag = *reinterpret_cast<volatile int*>(a.status) != 0;
    mbar_init(&bars->kv_full, 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&bars->qd_full[s], 1);
      mbar_init(&bars->qd_empty[s], 1);
    }
    mbar_init(&bars->st_full, 1);
    mbar_init(&bars->p_full, 128);
    mbar_init(&bars->dq_full, 1);
    mbar_init(&bars->dq_free, 128);
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
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      const int krb = jrank * g.B + b;
      mbar_expect_tx(&bars->kv_full, 2 * C::kTileBytes);
      for (int p = 0; p < C::kPanels; ++p) {
        tma_load_4d(&tm_k, &bars->kv_full, sK + p * C::kPanelBytes, p * 64, gl, k0, krb);
        tma_load_4d(&tm_v, &bars->kv_full, sV + p * C::kPanelBytes, p * 64, gl, k0, krb);
      }
      int issued = 0;
      for (QWalk qw = qwalk_begin(g, j, kmin, kmax); qw.valid; qwalk_next(g, j, kmin, kmax, qw), ++issued) {
        const int s = issued % C::kStages;
        if (issued >= C::kStages &&
            !mbar_wait(&bars->qd_empty[s], ((issued / C::kStages) - 1) & 1, w, kSiteBQdEmpty))
          break;
        const int h = gl * g.G + qw.hh;
        const int qrb = (qw.i * g.P_u + u) * g.B + b;
        const int q0 = qw.m * kBM;
        mbar_expect_tx(&bars->qd_full[s], 2 * C::kTileBytes + 1024);
        for (int p = 0; p < C::kPanels; ++p) {
          tma_load_4d(&tm_q, &bars->qd_full[s], sQ + s * C::kTileBytes + p * C::kPanelBytes, p * 64, h, q0, qrb);
          tma_load_4d(&tm_do, &bars->qd_full[s], sDO + s * C::kTileBytes + p * C::kPanelBytes, p * 64, h, q0,
                      qrb);
        }
        const size_t rowbase = (static_cast<size_t>(qrb) * g.Hq_l + h) * a.Lp + q0;
        bulk_load(sRow + s * 256, a.lse2 + rowbase, 512, &bars->qd_full[s]);
        bulk_load(sRow + s * 256 + 128, a.delta + rowbase, 512, &bars->qd_full[s]);
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
    if (lane == 0) {
      constexpr uint32_t kIdSS = idesc_bf16_f32(128, 128, 0, 0);  // both K-major
      constexpr uint32_t kIdKM = idesc_bf16_f32(128, D, 0, 1);    // A K-major, B MN-major
      constexpr uint32_t kIdMM = idesc_bf16_f32(128, D, 1, 1);    // both MN-major
      const uint32_t aK = smem_addr(sK), aV = smem_addr(sV), aQ = smem_addr(sQ), aDO = smem_addr(sDO);
      const uint32_t aPt = smem_addr(sPt), aDSt = smem_addr(sDSt);
      bool ok = mbar_wait(&bars->kv_full, 0, w, kSiteBKv);
      bool issued_any = false;
      int it = 0;
      for (QWalk qw = qwalk_begin(g, j, kmin, kmax); ok && qw.valid; qwalk_next(g, j, kmin, kmax, qw), ++it) {
        const int s = it % C::kStages;
        if (!mbar_wait(&bars->qd_full[s], (it / C::kStages) & 1, w, kSiteBQd)) { ok = false; break; }
        if (it >= 1 && !mbar_wait(&bars->dq_free, (it - 1) & 1, w, kSiteBDqFree)) { ok = false; break; }
        tc_fence_after();
        const uint32_t qb = aQ + s * C::kTileBytes, db = aDO + s * C::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::kPanelBytes + (kk & 3) * 32;
          umma_bf16(tmem + kColS, sdesc_sw128(aK + off, 16, 1024), sdesc_sw128(qb + off, 16, 1024), kIdSS,
                    kk > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::kPanelBytes + (kk & 3) * 32;
          umma_bf16(tmem + kColDP, sdesc_sw128(aV + off, 16, 1024), sdesc_sw128(db + off, 16, 1024), kIdSS,
                    kk > 0 ? 1u : 0u);
        }
        umma_commit(&bars->st_full);
        issued_any = true;
        if (!mbar_wait(&bars->p_full, it & 1, w, kSiteBP)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kBM / 16; ++kk) {  // K = 128 queries
          const uint32_t aoff = (kk >> 2) * C::kPanelBytes + (kk & 3) * 32;
          const uint32_t boff = kk * 16 * 128;
          umma_bf16(tmem + kColDV, sdesc_sw128(aPt + aoff, 16, 1024),
                    sdesc_sw128(db + boff, C::kPanelBytes, 1024), kIdKM, (it > 0 || kk > 0) ? 1u : 0u);
          umma_bf16(tmem + kColDK, sdesc_sw128(aDSt + aoff, 16, 1024),
                    sdesc_sw128(qb + boff, C::kPanelBytes, 1024), kIdKM, (it > 0 || kk > 0) ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {  // K = 128 keys
          const uint32_t off = kk * 16 * 128;
          umma_bf16(tmem + kColS, sdesc_sw128(aDSt + off, C::kPanelBytes, 1024),
                    sdesc_sw128(aK + off, C::kPanelBytes, 1024), kIdMM, kk > 0 ? 1u : 0u);
        }
        umma_commit(&bars->dq_full);
        umma_commit(&bars->qd_empty[s]);
      }
      if (!ok && issued_any) {
        umma_commit(&bars->drain);
        mbar_wait_drain(&bars->drain, 0, a.wait_ns);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ compute warps
    const int wq = warp & 3;
    const int row = wq * 32 + lane;  // key row of S^T / dP^T / dK / dV; query row of the dQ tile
    const uint32_t trow = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const int tau_k = k0 + row;
    const int pos_k = tau_k < g.L ? token_pos(g, j, tau_k) : INT_MAX;  // padding keys see no query
    const bool aligned = (g.c % kBM) == 0;
    bool ok = true;
    int it = 0;
    for (QWalk qw = qwalk_begin(g, j, kmin, kmax); qw.valid; qwalk_next(g, j, kmin, kmax, qw), ++it) {
      const int s = it % C::kStages;
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->st_full, it & 1, w, kSiteBSt));
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars->qd_full[s], (it / C::kStages) & 1, w, kSiteBQdC));
      if (!ok) break;
      tc_fence_after();
      const float* lse2 = sRow + s * 256;
      const float* dl = lse2 + 128;
      const int q0 = qw.m * kBM;
      const bool masked = qw.kind == kMasked;
      // Visible query columns: col >= lo (causal, aligned) and col < qvalid.
      int lo = 0;
      const int qvalid = g.L - q0;
      if (masked && aligned && g.causal) lo = pos_k == INT_MAX ? INT_MAX : pos_k - token_pos(g, qw.i, q0);
#pragma unroll
      for (int c0 = 0; c0 < kBM; c0 += 32) {
        uint32_t rs[32], rp[32];
        tmem_ld32(trow + kColS + c0, rs);
        tmem_ld32(trow + kColDP + c0, rp);
        tmem_ld_wait();
        reg_fence32(rs);
        reg_fence32(rp);
        uint32_t pk[16], dk[16];
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          float pv[2], dv[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int col = c0 + c + e;
            bool vis = true;
            if (masked) {
              if (aligned || !g.causal)
                vis = col >= lo && col < qvalid;
              else
                vis = col < qvalid && pos_k <= token_pos(g, qw.i, q0 + col);
            }
            const float p = vis ? ex2_approx(fmaf(__uint_as_float(rs[c + e]), g.scale_log2, -lse2[col])) : 0.f;
            pv[e] = p;
            dv[e] = p * (__uint_as_float(rp[c + e]) - dl[col]) * g.scale;
          }
          pk[c >> 1] = pack_bf16x2(pv[0], pv[1]);
          dk[c >> 1] = pack_bf16x2(dv[0], dv[1]);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int ch = (c0 >> 3) + q;  // 16-byte chunk index along the 128 queries
          const uint32_t off = (ch >> 3) * C::kPanelBytes + sw128_offset(row, ch & 7);
          *reinterpret_cast<uint4*>(sPt + off) = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
          *reinterpret_cast<uint4*>(sDSt + off) = make_uint4(dk[4 * q], dk[4 * q + 1], dk[4 * q + 2], dk[4 * q + 3]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&bars->p_full);
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->dq_full, it & 1, w, kSiteBDq));
      if (!ok) break;
      tc_fence_after();
      const int h = gl * g.G + qw.hh;
      const int qrank = qw.i * g.P_u + u;
      const bool add = q0 + row < g.L;
      float* dq_row = a.dq_acc + ((static_cast<size_t>(qrank * g.B + b) * g.L + (add ? q0 + row : 0)) * g.Hq_l + h) * D;
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(trow + kColS + c0, r);
        tmem_ld_wait();
        reg_fence32(r);
        if (add) {
#pragma unroll
          for (int q = 0; q < 8; ++q)
            atomicAdd(reinterpret_cast<float4*>(dq_row + c0) + q,
                      make_float4(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1]),
                                  __uint_as_float(r[4 * q + 2]), __uint_as_float(r[4 * q + 3])));
        }
      }
      tc_fence_before();
      mbar_arrive(&bars->dq_free);
    }
    // ------------------------------------------------------------ dK, dV epilogue
    if (ok) {
      tc_fence_after();
      const bool store = tau_k < g.L;
      const size_t kr = (static_cast<size_t>(jrank * g.B + b) * g.L + (store ? tau_k : 0)) * g.Hkv_l + gl;
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t rk[32], rv[32];
        if (it >= 1) {
          tmem_ld32(trow + kColDK + c0, rk);
          tmem_ld32(trow + kColDV + c0, rv);
          tmem_ld_wait();
          reg_fence32(rk);
          reg_fence32(rv);
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) rk[c] = rv[c] = 0u;
        }
        if (store) {
          float4* dkp = reinterpret_cast<float4*>(a.dk + kr * D + c0);
          float4* dvp = reinterpret_cast<float4*>(a.dv + kr * D + c0);
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            dkp[q] = make_float4(__uint_as_float(rk[4 * q]), __uint_as_float(rk[4 * q + 1]),
                                 __uint_as_float(rk[4 * q + 2]), __uint_as_float(rk[4 * q + 3]));
            dvp[q] = make_float4(__uint_as_float(rv[4 * q]), __uint_as_float(rv[4 * q + 1]),
                                 __uint_as_float(rv[4 * q + 2]), __uint_as_float(rv[4 * q + 3]));
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

template <int D>
cudaError_t launch_bwd_d(const BwdLaunch& L, cudaStream_t stream) {
  using C = BwdCfg<D>;
  static_assert(C::kSmemBytes <= 227 * 1024, "shared memory budget");
  cudaError_t e = cudaFuncSetAttribute(attn_bwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::kSmemBytes);
  if (e != cudaSuccess) return e;
  BwdArgs a{};
  a.g = make_geo(L.g);
  a.lse2 = L.lse2;
  a.delta = L.delta;
  a.Lp = L.Lp;
  a.dq_acc = L.dq_acc;
  a.dk = L.dk;
  a.dv = L.dv;
  a.status = L.status;
  a.wait_ns = L.wait_ns;
  const long long blocks = static_cast<long long>(a.g.n_ktiles) * a.g.n_ranks * a.g.B * a.g.Hkv_l;
  if (blocks <= 0) return cudaSuccess;
  if (blocks > 0x7FFFFFFFLL) return cudaErrorInvalidConfiguration;
  attn_bwd_kernel<D><<<static_cast<unsigned>(blocks), kThreadsBwd, C::kSmemBytes, stream>>>(L.tm_q, L.tm_k, L.tm_v,
                                                                                           L.tm_do, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_bwd(const BwdLaunch& L, cudaStream_t stream) {
  if (L.g.D == 128) return launch_bwd_d<128>(L, stream);
  if (L.g.D == 64) return launch_bwd_d<64>(L, stream);
  return cudaErrorInvalidValue;
}

}  // namespace usp
