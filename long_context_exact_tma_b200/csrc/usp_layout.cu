// usp_layout.cu -- bit-exact layout gathers: zigzag shard/unshard and the
// Ulysses seq<->head all-to-all emulated as on-device gathers.
//
// Zigzag (load balancing of the causal ring; "Boosting Spec Eagle",
// "Implementation Details"): 2P chunks of c tokens, rank r holds chunks r and
// 2P-1-r. Ulysses all-to-all (DeepSpeed-Ulysses summary, "Wie DeepSpeed-Ulysses
// funktioniert"): rank (i,u) receives head group u of every rank (i,u').
//
// Each kernel thread group walks DESTINATION runs ("pull"): a run is a
// contiguous row that is also contiguous in the source (a whole token of H
// heads for the zigzag maps, the H/P_u heads of one group for the all-to-all).
// Index math is done once per run, then the run is copied with 16-byte vectors
// (4-byte words when the run is not a multiple of 16 bytes, e.g. LSE rows).
// HBM-bound: 2 * tensor bytes of traffic per call.
#include "usp_internal.h"

namespace usp {
namespace {

struct RunMap {
  int map;
  uint32_t B, S, H, P_u, P_r;
  uint32_t P, c, c2, L, Hl;
  uint32_t run_bytes;  // bytes per run
  uint32_t n_runs;
  uint64_t row_bytes;  // bytes per head row
};

// Byte offsets (src, dst) of destination run q.
__device__ __forceinline__ void run_offsets(const RunMap& m, uint32_t q, uint64_t& so, uint64_t& dof) {
  switch (m.map) {
    case kZigzagShard: {  // dst rank-major token (r, b, t) <- global token (b, s)
      const uint32_t t = q % m.c2, rb = q / m.c2, b = rb % m.B, r = rb / m.B;
      const uint32_t s = t < m.c ? r * m.c + t : (2 * m.P - 1 - r) * m.c + (t - m.c);
      so = (static_cast<uint64_t>(b) * m.S + s) * m.run_bytes;
      dof = static_cast<uint64_t>(q) * m.run_bytes;
      break;
    }
    case kZigzagUnshard: {  // dst global token (b, s) <- rank-major token (r, b, t)
      const uint32_t s = q % m.S, b = q / m.S, chunk = s / m.c;
      const uint32_t r = chunk < m.P ? chunk : 2 * m.P - 1 - chunk;
      const uint32_t t = (chunk < m.P ? 0 : m.c) + s % m.c;
      so = (static_cast<uint64_t>(r * m.B + b) * m.c2 + t) * m.run_bytes;
      dof = static_cast<uint64_t>(q) * m.run_bytes;
      break;
    }
    case kSeq2Head: {  // dst (i,u,b,tau) head group <- rank (i,u'), token t, heads u*Hl..
      const uint32_t tau = q % m.L, q1 = q / m.L, b = q1 % m.B, iu = q1 / m.B;
      const uint32_t i = iu / m.P_u, u = iu % m.P_u;
      const uint32_t up = tau / m.c2, t = tau % m.c2, r = i * m.P_u + up;
      so = ((static_cast<uint64_t>(r * m.B + b) * m.c2 + t) * m.H + static_cast<uint64_t>(u) * m.Hl) * m.row_bytes;
      dof = static_cast<uint64_t>(q) * m.run_bytes;
      break;
    }
    default: {  // kHead2Seq: dst rank (r), b, t, head group u <- (i,u,b,tau)
      const uint32_t u = q % m.P_u, q1 = q / m.P_u, t = q1 % m.c2, rb = q1 / m.c2;
      const uint32_t b = rb % m.B, r = rb / m.B;
      const uint32_t i = r / m.P_u, up = r % m.P_u, tau = up * m.c2 + t;
      so = (static_cast<uint64_t>((i * m.P_u + u) * m.B + b) * m.L + tau) * m.run_bytes;
      dof = ((static_cast<uint64_t>(r * m.B + b) * m.c2 + t) * m.H + static_cast<uint64_t>(u) * m.Hl) * m.row_bytes;
      break;
    }
  }
}

template <typename V, int kUnroll>
__global__ void __launch_bounds__(256) layout_gather_kernel(const uint8_t* __restrict__ src,
                                                            uint8_t* __restrict__ dst, RunMap m,
                                                            uint32_t lanes_per_run) {
  const uint32_t lane = threadIdx.x & 31u;
  const uint32_t warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const uint32_t n_warps = (gridDim.x * blockDim.x) >> 5;
  const uint32_t runs_per_warp = 32u / lanes_per_run;
  const uint32_t sub = lane / lanes_per_run, sl = lane % lanes_per_run;
  const uint32_t nvec = m.run_bytes / sizeof(V);
  for (uint32_t q = warp * runs_per_warp + sub; q < m.n_runs; q += n_warps * runs_per_warp) {
    uint64_t so, dof;
    run_offsets(m, q, so, dof);
    const V* s = reinterpret_cast<const V*>(src + so);
    V* d = reinterpret_cast<V*>(dst + dof);
    for (uint32_t v0 = sl; v0 < nvec; v0 += kUnroll * lanes_per_run) {
      V buf[kUnroll];
#pragma unroll
      for (int k = 0; k < kUnroll; ++k) {
        const uint32_t v = v0 + k * lanes_per_run;
        if (v < nvec) buf[k] = __ldcs(s + v);
      }
#pragma unroll
      for (int k = 0; k < kUnroll; ++k) {
        const uint32_t v = v0 + k * lanes_per_run;
        if (v < nvec) __stcs(d + v, buf[k]);
      }
    }
  }
}

uint32_t pow2_at_least(uint32_t x) {
  uint32_t p = 1;
  while (p < x) p <<= 1;
  return p;
}

}  // namespace

cudaError_t launch_layout(const LayoutArgs& a, cudaStream_t stream) {
  RunMap m{};
  m.map = a.map;
  m.B = a.B; m.S = a.S; m.H = a.H; m.P_u = a.P_u; m.P_r = a.P_r;
  m.P = a.P_u * a.P_r;
  m.c = a.S / (2 * m.P);
  m.c2 = 2 * m.c;
  m.L = m.c2 * a.P_u;
  m.Hl = a.H / a.P_u;
  m.row_bytes = a.row_bytes;
  if (a.map == kZigzagShard || a.map == kZigzagUnshard) {
    m.run_bytes = a.H * a.row_bytes;
    m.n_runs = a.B * a.S;
  } else {
    m.run_bytes = m.Hl * a.row_bytes;
    m.n_runs = a.B * a.S * a.P_u;
  }
  if (m.n_runs == 0) return cudaSuccess;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // Every source and destination offset is a multiple of run_bytes (or of
  // H*row_bytes = P_u*run_bytes), so 16-byte runs keep 16-byte alignment.
  const bool vec16 = (m.run_bytes % 16 == 0) && (reinterpret_cast<uintptr_t>(a.src) % 16 == 0) &&
                     (reinterpret_cast<uintptr_t>(a.dst) % 16 == 0);
  const uint32_t nvec = m.run_bytes / (vec16 ? 16 : 4);
  const uint32_t lpr = nvec >= 32 ? 32 : pow2_at_least(nvec);
  const uint64_t threads_needed = static_cast<uint64_t>(m.n_runs) * lpr;
  uint64_t blocks = (threads_needed + 255) / 256;
  const uint64_t cap = static_cast<uint64_t>(sms) * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  if (vec16)
    layout_gather_kernel<uint4, 4><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(a.src, a.dst, m, lpr);
  else
    layout_gather_kernel<uint32_t, 4><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(a.src, a.dst, m, lpr);
  return cudaGetLastError();
}

}  // namespace usp
