// usp_attn_fwd.cu -- forward of exact softmax attention for every virtual rank
// of the USP mesh, block by block over the ring's KV chunks, on sm_100a.
//
// What it computes: for each ring rank i, Ulysses rank u, batch b, local query
// head h and 128-row query tile, the exact attention over the keys of every
// ring step t (owner j = (i - t) mod P_r), i.e. Ring Attention ("Boosting Spec
// Eagle", "The Solution") evaluated blockwise (Blockwise Parallel Transformer;
// LongNet slides, "Results": FlashAttention-style exact attention). The partial
// results of the ring steps are merged by log-sum-exp; in fused mode that merge
// happens online inside the kernel, in stepwise mode the kernel runs one ring
// step and writes the fp32 partial (O_t, LSE_t) for usp_lse_merge.
//
// CTA layout (192 threads, one 128-row query tile per CTA):
//   warp 0      TMA producer: Q once, then K and V tiles into a kStages ring.
//   warp 1      TMEM allocator and UMMA issuer (one thread):
//                 S[it&1] = Q K^T   (tcgen05.mma kind::f16, M=128 N=128, fp32 in TMEM)
//                 O      += P V     (M=128 N=D, A = P from shared memory)
//   warps 2..5  softmax: thread = query row = TMEM lane. Reads S with tcgen05.ld,
//               masks by original token positions, online max/sum in fp32 with
//               lazy rescaling of O (only when the row max grows by > 2^8),
//               writes P (bf16) into 128B-swizzled shared memory for the PV UMMA,
//               and finally normalises O and writes O (bf16) and LSE (fp32).
// TMEM columns: S0 [0,128), S1 [128,256), O [256, 256+D).
//
// Synchronisation is by mbarriers only; every wait is bounded (see usp_ptx.cuh).
#include <math.h>

#include "usp_attn_common.cuh"
#include "usp_internal.h"
#include "usp_ptx.cuh"

namespace usp {
namespace {

constexpr int kThreadsFwd = 192;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 256;
constexpr float kRescaleThresh = 8.0f;  // log2 units: rescale O only if the max grows by > 256x

template <int D>
struct FwdCfg {
  static constexpr int kPanels = D / 64;          // 128-byte (64 x bf16) swizzle panels along D
  static constexpr int kPanelBytes = 128 * 128;   // 128 rows x 128 bytes
  static constexpr int kTileBytes = kPanels * kPanelBytes;
  static constexpr int kStages = D == 128 ? 2 : 3;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kTileBytes;
  static constexpr int kOffV = kOffK + kStages * kTileBytes;
  static constexpr int kOffP = kOffV + kStages * kTileBytes;  // 128 x 128 bf16 = 2 panels
  static constexpr int kOffBar = kOffP + 2 * kPanelBytes;
  static constexpr int kSmemBytes = kOffBar + 512 + 1024;
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
};

struct FwdBars {
  uint64_t q_full;
  uint64_t k_full[3], v_full[3], kv_empty[3];
  uint64_t s_full[2], s_free[2];
  uint64_t p_full, o_done, drain;
  // Key-tile descriptors published by the producer with k_full of that tile:
  // {1, or -1 = no more tiles; ring rank j of the key owner; key tile n; tile kind}.
  int step[4][4];
  uint32_t tmem_base;
  int abort_flag;
};

// Wait-site codes recorded in the status word: 0x100 | role << 4 | which.
enum : int {
  kSiteQ = 0x101, kSiteKvEmpty = 0x102, kSiteK = 0x111, kSiteSFree = 0x112, kSiteP = 0x113, kSiteV = 0x114,
  kSiteS = 0x121, kSiteO = 0x122, kSiteKs = 0x123
};

template <int D>
__global__ void __launch_bounds__(kThreadsFwd, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const FwdArgs a) {
  using C = FwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  FwdBars* bars = reinterpret_cast<FwdBars*>(smem + C::kOffBar);
  uint8_t* sQ = smem + C::kOffQ;
  uint8_t* sK = smem + C::kOffK;
  uint8_t* sV = smem + C::kOffV;
  uint8_t* sP = smem + C::kOffP;

  const Geo& g = a.g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // Work item: CTAs of one (b, Ulysses rank, head) run together so that its K/V
  // stay in L2; inside it, query tiles in decreasing original position (the
  // causally heaviest first).
  const int n_qt = g.P_r * g.n_qtiles;
  int wi = blockIdx.x;
  const int order = n_qt - 1 - wi % n_qt;
  wi /= n_qt;
  const int h = wi % g.Hq_l;
  wi /= g.Hq_l;
  const int u = wi % g.P_u;
  const int b = wi / g.P_u;
  int i, m;
  tile_in_position_order(g, order, i, m);
  const int rank = i * g.P_u + u;
  const int kvh = h / g.G;
  const int q0 = m * kBM;
  const int t_begin = a.step < 0 ? 0 : a.step;
  const int t_end = a.step < 0 ? g.P_r : a.step + 1;
  int qmin, qmax;
  pos_range(g, i, q0, q0 + kBM, qmin, qmax);

  if (threadIdx.x == 0) {
    // A CTA that starts after another one gave up does no work at all.
    bars->abort_flag = *reinterpret_cast<volatile int*>(a.status) != 0;
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->s_full[s], 1);
      mbar_init(&bars->s_free[s], 128);
    }
    mbar_init(&bars->p_full, 128);
    mbar_init(&bars->o_done, 1);
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
  } else if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      KvWalk kw = kv_walk_begin(g, i, qmin, qmax, t_begin, t_end);
      int issued = 0;
      const bool any = kw.valid;
      {
        if (any) {
          tma_prefetch_desc(&tm_q);
          tma_prefetch_desc(&tm_k);
          tma_prefetch_desc(&tm_v);
          mbar_expect_tx(&bars->q_full, C::kTileBytes);
          for (int p = 0; p < C::kPanels; ++p)
            tma_load_4d(&tm_q, &bars->q_full, sQ + p * C::kPanelBytes, p * 64, h, q0, rank * g.B + b);
        }
        while (true) {
          const int s = issued % C::kStages;
          if (issued >= C::kStages &&
              !mbar_wait(&bars->kv_empty[s], ((issued / C::kStages) - 1) & 1, w, kSiteKvEmpty))
            break;
          int* slot = bars->step[issued & 3];
          if (!kw.valid) {  // publish the end of the walk on this stage's barrier
            slot[0] = -1;
            mbar_arrive(&bars->k_full[s]);
            break;
          }
          slot[0] = 1;
          slot[1] = kw.j;
          slot[2] = kw.n;
          slot[3] = kw.kind;
          const int krb = (kw.j * g.P_u + u) * g.B + b;
          mbar_expect_tx(&bars->k_full[s], C::kTileBytes);
          for (int p = 0; p < C::kPanels; ++p)
            tma_load_4d(&tm_k, &bars->k_full[s], sK + s * C::kTileBytes + p * C::kPanelBytes, p * 64, kvh,
                        kw.n * kBN, krb);
          mbar_expect_tx(&bars->v_full[s], C::kTileBytes);
          for (int p = 0; p < C::kPanels; ++p)
            tma_load_4d(&tm_v, &bars->v_full[s], sV + s * C::kTileBytes + p * C::kPanelBytes, p * 64, kvh,
                        kw.n * kBN, krb);
          ++issued;
          kv_walk_next(g, i, qmin, qmax, t_end, kw);
        }
        if (*reinterpret_cast<volatile int*>(&bars->abort_flag)) {
          // Let every copy this thread started land before the CTA exits.
          if (any) mbar_wait_drain(&bars->q_full, 0, a.wait_ns);
          for (int it = issued - C::kStages < 0 ? 0 : issued - C::kStages; it < issued; ++it) {
            mbar_wait_drain(&bars->k_full[it % C::kStages], (it / C::kStages) & 1, a.wait_ns);
            mbar_wait_drain(&bars->v_full[it % C::kStages], (it / C::kStages) & 1, a.wait_ns);
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ UMMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdescQK = idesc_bf16_f32(kBM, kBN, 0, 0);
      constexpr uint32_t kIdescPV = idesc_bf16_f32(kBM, D, 0, 1);
      const uint32_t aQ = smem_addr(sQ), aK = smem_addr(sK), aV = smem_addr(sV), aP = smem_addr(sP);
      bool ok = true;
      int it = 0;
      bool issued_any = false;
      auto issue_pv = [&](int p) -> bool {
        const int s = p % C::kStages;
        if (!mbar_wait(&bars->p_full, p & 1, w, kSiteP)) return false;
        if (!mbar_wait(&bars->v_full[s], (p / C::kStages) & 1, w, kSiteV)) return false;
        tc_fence_after();
        const uint32_t vbase = aV + s * C::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          const uint64_t da = sdesc_sw128(aP + (kk >> 2) * C::kPanelBytes + (kk & 3) * 32, 16, 1024);
          const uint64_t db = sdesc_sw128(vbase + kk * 16 * 128, C::kPanelBytes, 1024);
          umma_bf16(tmem + kColO, da, db, kIdescPV, (p > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&bars->o_done);
        umma_commit(&bars->kv_empty[s]);
        return true;
      };
      ok = mbar_wait(&bars->k_full[0], 0, w, kSiteK);
      bool have = ok && bars->step[0][0] >= 0;
      if (have) ok = mbar_wait(&bars->q_full, 0, w, kSiteQ);
      for (; ok && have; ++it) {
        const int s = it % C::kStages;
        const int sb = it & 1;
        if (it > 0) {
          if (!mbar_wait(&bars->k_full[s], (it / C::kStages) & 1, w, kSiteK)) { ok = false; break; }
          if (bars->step[it & 3][0] < 0) break;
        }
        if (it >= 2 && !mbar_wait(&bars->s_free[sb], ((it >> 1) - 1) & 1, w, kSiteSFree)) { ok = false; break; }
        tc_fence_after();
        const uint32_t kbase = aK + s * C::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::kPanelBytes + (kk & 3) * 32;
          umma_bf16(tmem + sb * 128, sdesc_sw128(aQ + off, 16, 1024), sdesc_sw128(kbase + off, 16, 1024),
                    kIdescQK, kk > 0 ? 1u : 0u);
        }
        umma_commit(&bars->s_full[sb]);
        issued_any = true;
        if (it >= 1 && !issue_pv(it - 1)) { ok = false; break; }
      }
      if (ok && it >= 1) ok = issue_pv(it - 1);
      if (!ok && issued_any) {
        umma_commit(&bars->drain);
        mbar_wait_drain(&bars->drain, 0, a.wait_ns);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax warps
    const int wq = warp & 3;  // TMEM lane quarter of this warp
    const int row = wq * 32 + lane;
    const uint32_t trow = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const int tau_q = q0 + row;
    const int pos_q = tau_q < g.L ? token_pos(g, i, tau_q) : INT_MAX;
    const bool aligned = (g.c % kBN) == 0;
    // l_run: sum of the fp32 weights (for LSE); lb_run: sum of the bf16-rounded
    // weights the PV UMMA consumes (normalises O, so O stays a convex combination
    // of V rows even when one key dominates).
    float m_use = -INFINITY, l_run = 0.f, lb_run = 0.f;
    int it = 0;
    bool ok = true;
    for (;; ++it) {
      const int sb = it & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->k_full[it % C::kStages], (it / C::kStages) & 1, w, kSiteKs));
      if (!ok) break;
      const int* slot = bars->step[it & 3];
      if (slot[0] < 0) break;
      const int kj = slot[1], kn = slot[2], kkind = slot[3];
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->s_full[sb], (it >> 1) & 1, w, kSiteS));
      if (!ok) break;
      tc_fence_after();
      uint32_t r0[32], r1[32], r2[32], r3[32];
      tmem_ld32(trow + sb * 128 + 0, r0);
      tmem_ld32(trow + sb * 128 + 32, r1);
      tmem_ld32(trow + sb * 128 + 64, r2);
      tmem_ld32(trow + sb * 128 + 96, r3);
      tmem_ld_wait();
      reg_fence32(r0);
      reg_fence32(r1);
      reg_fence32(r2);
      reg_fence32(r3);
      tc_fence_before();
      mbar_arrive(&bars->s_free[sb]);
      float s[128];
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        s[c] = __uint_as_float(r0[c]);
        s[32 + c] = __uint_as_float(r1[c]);
        s[64 + c] = __uint_as_float(r2[c]);
        s[96 + c] = __uint_as_float(r3[c]);
      }
      if (kkind == kMasked) {
        const int k0 = kn * kBN;
        const int kvalid = g.L - k0;  // keys at or past this column are padding
        if (aligned) {
          // the whole key tile lies in one chunk: positions are base + column
          const int lim = g.causal ? pos_q - token_pos(g, kj, k0) : INT_MAX;
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c > lim || c >= kvalid) s[c] = -INFINITY;
        } else {
#pragma unroll
          for (int c = 0; c < 128; ++c) {
            const bool vis = c < kvalid && (!g.causal || token_pos(g, kj, k0 + c) <= pos_q);
            if (!vis) s[c] = -INFINITY;
          }
        }
      }
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 128; ++c) mx = fmaxf(mx, s[c]);
      const float m_tile = mx * g.scale_log2;
      const bool bump = m_tile > m_use + kRescaleThresh;
      float alpha = 1.f;
      if (bump) {
        alpha = ex2_approx(m_use - m_tile);
        m_use = m_tile;
      }
      const float m_safe = m_use == -INFINITY ? 0.f : m_use;
      float rs = 0.f;
#pragma unroll
      for (int c = 0; c < 128; ++c) {
        s[c] = ex2_approx(fmaf(s[c], g.scale_log2, -m_safe));
        rs += s[c];
      }
      l_run = l_run * alpha + rs;
      lb_run *= alpha;
      if (it >= 1) {
        ok = __all_sync(0xffffffffu, mbar_wait(&bars->o_done, (it - 1) & 1, w, kSiteO));
        if (!ok) break;
        tc_fence_after();
        if (__any_sync(0xffffffffu, bump)) {
#pragma unroll
          for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t o[32];
            tmem_ld32(trow + kColO + c0, o);
            tmem_ld_wait();
            reg_fence32(o);
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
            tmem_st32(trow + kColO + c0, o);
          }
          tmem_st_wait();
        }
      }
      // P (bf16) into the two 64-key swizzled panels, row = query row.
      float rsb = 0.f;
#pragma unroll
      for (int ch = 0; ch < 16; ++ch) {
        uint4 v;
        v.x = pack_bf16x2(s[ch * 8 + 0], s[ch * 8 + 1]);
        v.y = pack_bf16x2(s[ch * 8 + 2], s[ch * 8 + 3]);
        v.z = pack_bf16x2(s[ch * 8 + 4], s[ch * 8 + 5]);
        v.w = pack_bf16x2(s[ch * 8 + 6], s[ch * 8 + 7]);
        rsb += bf16x2_sum(v.x) + bf16x2_sum(v.y) + bf16x2_sum(v.z) + bf16x2_sum(v.w);
        *reinterpret_cast<uint4*>(sP + (ch >> 3) * C::kPanelBytes + sw128_offset(row, ch & 7)) = v;
      }
      lb_run += rsb;
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&bars->p_full);
    }
    // ------------------------------------------------------------ epilogue
    if (ok && it >= 1) ok = __all_sync(0xffffffffu, mbar_wait(&bars->o_done, (it - 1) & 1, w, kSiteO));
    if (ok) {
      tc_fence_after();
      const bool store = tau_q < g.L;
      const size_t row_idx = (static_cast<size_t>(rank * g.B + b) * g.L + (store ? tau_q : 0)) * g.Hq_l + h;
      const float inv_l = lb_run > 0.f ? 1.f / lb_run : 0.f;
      const float lse_val = l_run > 0.f ? (m_use + __log2f(l_run)) * 0.6931471805599453f : -INFINITY;
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t o[32];
        if (it >= 1) {
          tmem_ld32(trow + kColO + c0, o);
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
            for (int q = 0; q < 8; ++q)
              dst[q] = make_float4(__uint_as_float(o[q * 4 + 0]) * inv_l, __uint_as_float(o[q * 4 + 1]) * inv_l,
                                   __uint_as_float(o[q * 4 + 2]) * inv_l, __uint_as_float(o[q * 4 + 3]) * inv_l);
          }
        }
      }
      if (store) {
        if (a.step < 0)
          a.lse[row_idx] = lse_val;
        else
          a.lse_part[row_idx] = lse_val;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D>
cudaError_t launch_fwd_d(const FwdLaunch& L, cudaStream_t stream) {
  using C = FwdCfg<D>;
  static_assert(C::kSmemBytes <= 227 * 1024, "shared memory budget");
  cudaError_t e = cudaFuncSetAttribute(attn_fwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::kSmemBytes);
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
  const long long blocks = static_cast<long long>(a.g.n_qtiles) * a.g.n_ranks * a.g.B * a.g.Hq_l;
  if (blocks <= 0) return cudaSuccess;
  if (blocks > 0x7FFFFFFFLL) return cudaErrorInvalidConfiguration;
  attn_fwd_kernel<D><<<static_cast<unsigned>(blocks), kThreadsFwd, C::kSmemBytes, stream>>>(L.tm_q, L.tm_k,
                                                                                           L.tm_v, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_fwd(const FwdLaunch& L, cudaStream_t stream) {
  if (L.g.D == 128) return launch_fwd_d<128>(L, stream);
  if (L.g.D == 64) return launch_fwd_d<64>(L, stream);
  return cudaErrorInvalidValue;
}

}  // namespace usp
