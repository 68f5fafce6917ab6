// usp_layout.cu -- bit-exact layout gathers: zigzag shard/unshard and the
// Ulysses seq<->head all-to-all emulated as on-device gathers.
//
// Zigzag (load balancing of the causal ring; "Boosting Spec Eagle",
// "Implementation Details"): 2P chunks of c tokens, rank r holds chunks r and
// 2P-1-r. Ulysses all-to-all (DeepSpeed-Ulysses summary, "Wie DeepSpeed-Ulysses
// funktioniert"): rank (i,u) receives head group u of every rank (i,u').
//
// The kernel walks DESTINATION runs ("pull"): a run is a contiguous row that is
// also contiguous in the source (a whole token of H heads for the zigzag maps,
// the H/P_u heads of one group for the all-to-all). One launch may move up to
// kMaxLayoutJobs tensors with the same map and mesh (Q, K, V of a step; or dQ, dK,
// dV), so launch and tail are paid once.
//
// Work is split into warp tasks of (nearly) equal size, four vectors per lane:
// a long run is cut into pieces of 128 vectors (each group of 32 lanes reading
// 512 contiguous bytes), shorter runs are packed several to a task. Warp w
// takes tasks w, w + W, ... (W warps in the grid) two at a time, with all their
// loads in flight before the stores, so that no warp has more than one task
// more than another whatever the run length. The index math of a task is done
// once, for its first run. HBM-bound: 2 x tensor bytes per job.
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

struct Job {
  const uint8_t* src;
  uint8_t* dst;
  RunMap m;
  uint32_t nvec;        // vectors per run
  uint32_t lanes;       // lanes per run (32 for long and medium runs)
  uint32_t pieces;      // tasks per run (long runs); 0 otherwise
  uint32_t xslots;      // slots per run (medium runs)
  uint32_t runs_per_task;
  uint32_t seg;         // runs per contiguous source segment
  uint64_t src_step;    // source bytes between consecutive runs of a segment
  uint32_t task_begin;  // first flat task index of this job
};

struct Batch {
  Job job[kMaxLayoutJobs];
  int n_jobs;
  uint32_t n_tasks;
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
    case kPackHeads: {  // dst (g, b, t) <- src (b, t, g)
      const uint32_t t = q % m.S, q1 = q / m.S, b = q1 % m.B, gg = q1 / m.B;
      so = (static_cast<uint64_t>(b * m.S + t) * m.P_u + gg) * m.run_bytes;
      dof = static_cast<uint64_t>(q) * m.run_bytes;
      break;
    }
    case kUnpackHeads: {  // dst (b, t, g) <- src (g, b, t)
      const uint32_t gg = q % m.P_u, q1 = q / m.P_u, t = q1 % m.S, b = q1 / m.S;
      so = (static_cast<uint64_t>(gg * m.B + b) * m.S + t) * m.run_bytes;
      dof = static_cast<uint64_t>(q) * m.run_bytes;
      break;
    }
    case kPackTokens: {  // dst (g, b, t) <- src (b, g, t)
      const uint32_t t = q % m.S, q1 = q / m.S, b = q1 % m.B, gg = q1 / m.B;
      so = (static_cast<uint64_t>(b * m.P_u + gg) * m.S + t) * m.run_bytes;
      dof = static_cast<uint64_t>(q) * m.run_bytes;
      break;
    }
    case kUnpackTokens: {  // dst (b, g, t) <- src (g, b, t)
      const uint32_t t = q % m.S, q1 = q / m.S, gg = q1 % m.P_u, b = q1 / m.P_u;
      so = (static_cast<uint64_t>(gg * m.B + b) * m.S + t) * m.run_bytes;
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

constexpr int kSlots = 4;  // vectors a lane moves per task (one per slot)

// Where this lane's vectors of flat task `task` are. A task is kSlots slots of
// one 16-byte (or 4-byte) vector per lane:
//   long runs (>= 128 vectors): slot x is vector piece*128 + 32x + lane of one run;
//   medium runs (32..127 vectors): X = ceil(nvec/32) slots per run, 4/X runs;
//   short runs (< 32 vectors): `lanes` lanes per run, 32/lanes runs per slot.
// The offsets of a task's first run are computed once; the next runs of the
// task lie `src_step` / run_bytes further on while they stay in the same
// contiguous source segment of `seg` runs, else they are computed afresh.
template <typename V>
__device__ __forceinline__ void task_lane(const Batch& bt, uint32_t task, uint32_t lane, const V* (&s)[kSlots],
                                          V* (&d)[kSlots]) {
  int k = 0;
#pragma unroll
  for (int x = 1; x < kMaxLayoutJobs; ++x)
    if (x < bt.n_jobs && task >= bt.job[x].task_begin) k = x;
  const Job& jb = bt.job[k];
  const uint32_t local = task - jb.task_begin;
  if (jb.pieces > 0) {
    const uint32_t run = local / jb.pieces;
    const uint32_t v0 = (local % jb.pieces) * (32 * kSlots) + lane;
    uint64_t so, dof;
    run_offsets(jb.m, run, so, dof);
    const V* sp = reinterpret_cast<const V*>(jb.src + so);
    V* dp = reinterpret_cast<V*>(jb.dst + dof);
#pragma unroll
    for (int x = 0; x < kSlots; ++x) {
      const uint32_t vec = v0 + 32 * x;
      s[x] = vec < jb.nvec ? sp + vec : nullptr;
      d[x] = dp + vec;
    }
    return;
  }
  const uint32_t q0 = local * jb.runs_per_task;
  uint64_t so0, dof0;
  run_offsets(jb.m, q0, so0, dof0);
  const uint32_t in_seg = q0 % jb.seg;
  const bool medium = jb.lanes == 32;
#pragma unroll
  for (int x = 0; x < kSlots; ++x) {
    uint32_t dq, vec;
    bool ok;
    if (medium) {
      dq = x / jb.xslots;
      vec = (x % jb.xslots) * 32 + lane;
      ok = dq < jb.runs_per_task;
    } else {
      dq = x * (32 / jb.lanes) + lane / jb.lanes;
      vec = lane % jb.lanes;
      ok = true;
    }
    const uint32_t q = q0 + dq;
    ok = ok && q < jb.m.n_runs && vec < jb.nvec;
    s[x] = nullptr;
    d[x] = nullptr;
    if (ok) {
      uint64_t so, dof;
      if (in_seg + dq < jb.seg) {
        so = so0 + static_cast<uint64_t>(dq) * jb.src_step;
        dof = dof0 + static_cast<uint64_t>(dq) * jb.m.run_bytes;
      } else {
        run_offsets(jb.m, q, so, dof);
      }
      s[x] = reinterpret_cast<const V*>(jb.src + so) + vec;
      d[x] = reinterpret_cast<V*>(jb.dst + dof) + vec;
    }
  }
}

template <typename V>
__global__ void __launch_bounds__(256) layout_gather_kernel(const __grid_constant__ Batch bt) {
  constexpr int kTasks = 2;  // tasks per warp in flight
  const uint32_t lane = threadIdx.x & 31u;
  const uint32_t warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const uint32_t n_warps = (gridDim.x * blockDim.x) >> 5;
  for (uint32_t t0 = warp; t0 < bt.n_tasks; t0 += kTasks * n_warps) {
    V buf[kTasks][kSlots];
    V* dst[kTasks][kSlots];
#pragma unroll
    for (int y = 0; y < kTasks; ++y) {
      const uint32_t task = t0 + y * n_warps;
      const V* src[kSlots];
      if (task < bt.n_tasks) {
        task_lane<V>(bt, task, lane, src, dst[y]);
      } else {
#pragma unroll
        for (int x = 0; x < kSlots; ++x) src[x] = nullptr;
      }
#pragma unroll
      for (int x = 0; x < kSlots; ++x) {
        if (src[x] != nullptr) buf[y][x] = __ldcs(src[x]);
        if (src[x] == nullptr) dst[y][x] = nullptr;
      }
    }
#pragma unroll
    for (int y = 0; y < kTasks; ++y)
#pragma unroll
      for (int x = 0; x < kSlots; ++x)
        if (dst[y][x] != nullptr) __stcs(dst[y][x], buf[y][x]);
  }
}

uint32_t pow2_at_least(uint32_t x) {
  uint32_t p = 1;
  while (p < x) p <<= 1;
  return p;
}

RunMap make_map(int map, uint32_t B, uint32_t S, uint32_t H, uint32_t P_u, uint32_t P_r, uint32_t row_bytes) {
  RunMap m{};
  m.map = map;
  m.B = B; m.S = S; m.H = H; m.P_u = P_u; m.P_r = P_r;
  m.P = P_u * P_r;
  m.c = S / (2 * m.P);
  m.c2 = 2 * m.c;
  m.L = m.c2 * P_u;
  m.Hl = H / P_u;
  m.row_bytes = row_bytes;
  if (map == kZigzagShard || map == kZigzagUnshard) {
    m.run_bytes = H * row_bytes;
    m.n_runs = B * S;
  } else if (map >= kPackHeads) {  // S = T tokens per rank, P_u = G ranks
    m.run_bytes = m.Hl * row_bytes;
    m.n_runs = B * S * P_u;
  } else {
    m.run_bytes = m.Hl * row_bytes;
    m.n_runs = B * S * P_u;
  }
  return m;
}

}  // namespace

cudaError_t launch_layout_batch(const LayoutArgs* a, int n, cudaStream_t stream) {
  if (n <= 0 || n > kMaxLayoutJobs) return cudaErrorInvalidValue;
  Batch bt{};
  bt.n_jobs = n;
  // 16-byte vectors when every run of every job starts on a 16-byte boundary:
  // every source and destination offset is a multiple of run_bytes (or of
  // H*row_bytes = P_u*run_bytes), so 16-byte runs on 16-byte bases qualify.
  bool vec16 = true;
  for (int x = 0; x < n; ++x) {
    bt.job[x].m = make_map(a[x].map, a[x].B, a[x].S, a[x].H, a[x].P_u, a[x].P_r, a[x].row_bytes);
    vec16 = vec16 && bt.job[x].m.run_bytes % 16 == 0 && reinterpret_cast<uintptr_t>(a[x].src) % 16 == 0 &&
            reinterpret_cast<uintptr_t>(a[x].dst) % 16 == 0;
  }
  const uint32_t vsz = vec16 ? 16 : 4;
  uint64_t tasks = 0;
  for (int x = 0; x < n; ++x) {
    Job& jb = bt.job[x];
    jb.src = a[x].src;
    jb.dst = a[x].dst;
    jb.nvec = jb.m.run_bytes / vsz;
    jb.task_begin = static_cast<uint32_t>(tasks);
    const RunMap& m = jb.m;
    // contiguous source segments of consecutive destination runs
    switch (m.map) {
      case kZigzagShard:
      case kZigzagUnshard: jb.seg = m.c; jb.src_step = m.run_bytes; break;
      case kSeq2Head: jb.seg = m.c2; jb.src_step = static_cast<uint64_t>(m.H) * m.row_bytes; break;
      case kPackHeads: jb.seg = m.S; jb.src_step = static_cast<uint64_t>(m.P_u) * m.run_bytes; break;
      case kUnpackHeads: jb.seg = m.P_u; jb.src_step = static_cast<uint64_t>(m.B) * m.S * m.run_bytes; break;
      case kPackTokens:
      case kUnpackTokens: jb.seg = m.S; jb.src_step = m.run_bytes; break;
      default: jb.seg = m.P_u; jb.src_step = static_cast<uint64_t>(m.B) * m.L * m.run_bytes; break;
    }
    if (jb.nvec >= 32 * kSlots) {
      jb.lanes = 32;
      jb.pieces = (jb.nvec + 32 * kSlots - 1) / (32 * kSlots);
      jb.xslots = 0;
      jb.runs_per_task = 1;
      tasks += static_cast<uint64_t>(m.n_runs) * jb.pieces;
    } else {
      jb.pieces = 0;
      if (jb.nvec >= 32) {
        jb.lanes = 32;
        jb.xslots = (jb.nvec + 31) / 32;
        jb.runs_per_task = kSlots / jb.xslots;
      } else {
        jb.lanes = pow2_at_least(jb.nvec);
        jb.xslots = 1;
        jb.runs_per_task = kSlots * (32 / jb.lanes);
      }
      tasks += (static_cast<uint64_t>(m.n_runs) + jb.runs_per_task - 1) / jb.runs_per_task;
    }
  }
  if (tasks == 0) return cudaSuccess;
  if (tasks >= (1ull << 32) - (1ull << 28)) return cudaErrorInvalidValue;
  bt.n_tasks = static_cast<uint32_t>(tasks);
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // 8 CTAs of 8 warps per SM (the SM's full 2048 threads), fewer when there are
  // fewer tasks: each warp then takes an equal share of the tasks.
  uint64_t blocks = (tasks + 7) / 8;
  const uint64_t cap = static_cast<uint64_t>(sms) * 8;
  if (blocks > cap) blocks = cap;
  if (vec16)
    layout_gather_kernel<uint4><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(bt);
  else
    layout_gather_kernel<uint32_t><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(bt);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_layout(const LayoutArgs& a, cudaStream_t stream) { return launch_layout_batch(&a, 1, stream); }

}  // namespace usp
