// usp_elementwise.cu -- HBM-bound kernels around the attention kernels:
//   * log-sum-exp merge of ring-step partials (per ring step each rank holds a
//     partial (O_t, LSE_t) of its queries; "Boosting Spec Eagle", "The Solution",
//     Ring Attention),
//   * backward preprocess Delta_i = sum_d dO_id O_id,
//   * the bounded-wait self-test kernel.
#include <math.h>

#include "usp_internal.h"
#include "usp_ptx.cuh"

namespace usp {
namespace {

// One warp per row; lane l handles elements 4l, 4l+1, 4l+2, 4l+3 (+128 per pass).
// The output may alias partial 0 (out == o_parts, lse_out == lse_parts): the
// streamed ring merge folds each step into the running result in place. Every
// element is read and then written by the same lane, and the row's LSE is
// written only after the whole warp has read the partial LSEs (plain coherent
// loads, no restrict: the buffers may overlap).
template <bool kOutF32>
__global__ void __launch_bounds__(256) lse_merge_kernel(const float* o_parts, const float* lse_parts, int n_parts,
                                                        long long rows, int D, void* out, float* lse_out) {
  const int lane = threadIdx.x & 31;
  const long long n_warps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  for (long long r = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; r < rows;
       r += n_warps) {
    float m = -INFINITY;
    for (int t = 0; t < n_parts; ++t) m = fmaxf(m, lse_parts[static_cast<long long>(t) * rows + r]);
    float lse = -INFINITY;
    if (m != -INFINITY) {
      float acc = 0.f;
      for (int t = 0; t < n_parts; ++t) acc += expf(lse_parts[static_cast<long long>(t) * rows + r] - m);
      lse = m + logf(acc);
    }
    for (int d4 = lane; d4 * 4 < D; d4 += 32) {
      float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
      if (lse != -INFINITY) {
        for (int t = 0; t < n_parts; ++t) {
          const float lt = lse_parts[static_cast<long long>(t) * rows + r];
          if (lt == -INFINITY) continue;
          const float w = expf(lt - lse);
          const float4 p = __ldcs(reinterpret_cast<const float4*>(o_parts + (static_cast<long long>(t) * rows + r) * D) + d4);
          o.x += w * p.x;
          o.y += w * p.y;
          o.z += w * p.z;
          o.w += w * p.w;
        }
      }
      if (kOutF32) {
        reinterpret_cast<float4*>(static_cast<float*>(out) + r * D)[d4] = o;
      } else {
        uint2 packed;
        packed.x = pack_bf16x2(o.x, o.y);
        packed.y = pack_bf16x2(o.z, o.w);
        reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(out) + r * D)[d4] = packed;
      }
    }
    __syncwarp();
    if (lane == 0) lse_out[r] = lse;
  }
}

// The merge of one or two partials with D <= 128 (the streamed ring merge: the
// running result and one step's partial): every load of a row -- its partial
// LSEs and its lane's float4 of each partial O -- is issued before any of them
// is used, so a row costs one memory round trip. Alias-safe like the general
// kernel above (out may be partial 0).
template <bool kOutF32, int kN>
__global__ void __launch_bounds__(256) lse_merge_small_kernel(const float* o_parts, const float* lse_parts,
                                                              long long rows, int D, void* out, float* lse_out) {
  const int lane = threadIdx.x & 31;
  const bool active = lane * 4 < D;
  const long long n_warps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  for (long long r = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; r < rows;
       r += n_warps) {
    float lt[kN];
    float4 p[kN];
#pragma unroll
    for (int t = 0; t < kN; ++t) {
      lt[t] = lse_parts[static_cast<long long>(t) * rows + r];
      p[t] = active ? __ldcs(reinterpret_cast<const float4*>(o_parts + (static_cast<long long>(t) * rows + r) * D) +
                             lane)
                    : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float m = lt[0];
#pragma unroll
    for (int t = 1; t < kN; ++t) m = fmaxf(m, lt[t]);
    float lse = -INFINITY;
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
    if (m != -INFINITY) {
      float acc = 0.f;
#pragma unroll
      for (int t = 0; t < kN; ++t) acc += expf(lt[t] - m);
      lse = m + logf(acc);
#pragma unroll
      for (int t = 0; t < kN; ++t) {
        if (lt[t] == -INFINITY) continue;
        const float w = expf(lt[t] - lse);
        o.x += w * p[t].x;
        o.y += w * p[t].y;
        o.z += w * p[t].z;
        o.w += w * p[t].w;
      }
    }
    if (active) {
      if (kOutF32) {
        reinterpret_cast<float4*>(static_cast<float*>(out) + r * D)[lane] = o;
      } else {
        uint2 packed;
        packed.x = pack_bf16x2(o.x, o.y);
        packed.y = pack_bf16x2(o.z, o.w);
        reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(out) + r * D)[lane] = packed;
      }
    }
    __syncwarp();
    if (lane == 0) lse_out[r] = lse;
  }
}

// dO_r . O_r of one row of D bf16 (16-byte read-only loads: when the rows of a
// warp's threads lie apart, the second half of each 32-byte sector comes from L1).
__device__ __forceinline__ float row_dot_bf16(const __nv_bfloat16* a, const __nv_bfloat16* b, int D) {
  const uint4* pa = reinterpret_cast<const uint4*>(a);
  const uint4* pb = reinterpret_cast<const uint4*>(b);
  float acc0 = 0.f, acc1 = 0.f;
#pragma unroll 4
  for (int c = 0; c < D / 8; ++c) {
    const uint4 x = __ldg(pa + c), y = __ldg(pb + c);
    const __nv_bfloat162* x2 = reinterpret_cast<const __nv_bfloat162*>(&x);
    const __nv_bfloat162* y2 = reinterpret_cast<const __nv_bfloat162*>(&y);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 fx = __bfloat1622float2(x2[k]);
      const float2 fy = __bfloat1622float2(y2[k]);
      acc0 = fmaf(fx.x, fy.x, acc0);
      acc1 = fmaf(fx.y, fy.y, acc1);
    }
  }
  return acc0 + acc1;
}

// Delta_r = dO_r . O_r, thread per row.
__global__ void __launch_bounds__(256) bwd_preprocess_kernel(const __nv_bfloat16* __restrict__ out,
                                                             const __nv_bfloat16* __restrict__ dO,
                                                             float* __restrict__ delta, long long rows, int D) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long r = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; r < rows; r += stride)
    delta[r] = row_dot_bf16(out + r * D, dO + r * D, D);
}

// The per-head tables of the backward kernels, thread per row: consecutive threads
// take consecutive rows tau of one (rank-batch, head), so their -Delta and
// -LSE*log2(e) entries are written side by side.
__global__ void __launch_bounds__(256) bwd_prep_rows_kernel(const __nv_bfloat16* __restrict__ out,
                                                            const __nv_bfloat16* __restrict__ dO,
                                                            const float* __restrict__ lse,
                                                            float* __restrict__ delta_t, float* __restrict__ lse2_t,
                                                            long long rows, int L, int Hl, int D, int Lp) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long x = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; x < rows; x += stride) {
    const long long tau = x % L, hb = x / L;  // hb = rank-batch * Hl + head
    const long long r = ((hb / Hl) * L + tau) * Hl + hb % Hl;
    const long long dst = hb * Lp + tau;
    delta_t[dst] = -row_dot_bf16(out + r * D, dO + r * D, D);
    // a row that saw no key (LSE = -inf, O = 0; masked attention) must give
    // P = 0, as the padding rows do, not exp2(+inf)
    const float l = lse[r];
    lse2_t[dst] = l == -INFINITY ? -INFINITY : -l * 1.4426950408889634f;
  }
  // Padding rows [L, Lp) of every head: LSE = +inf and Delta = 0, so a padded
  // query contributes exactly zero (P = exp2(s - inf) = 0) whatever the workspace held.
  const long long pad = Lp - L;
  if (pad > 0) {
    const long long n_pad = (rows / L) * pad;  // heads * padding rows
    const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
    for (long long x = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; x < n_pad; x += stride) {
      const long long dst = (x / pad) * Lp + L + x % pad;
      delta_t[dst] = 0.f;
      lse2_t[dst] = -INFINITY;
    }
  }
}

// The empty running result of a merge: O = 0 (rows x D) and LSE = -inf (rows).
__global__ void __launch_bounds__(256) fill_running_kernel(float4* __restrict__ o, float* __restrict__ lse,
                                                           long long n4, long long rows) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long x = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; x < n4; x += stride)
    o[x] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (long long x = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; x < rows; x += stride)
    lse[x] = -INFINITY;
}

// Row tables of one dilated-attention backward launch: for problem p (batch
// p / n_seg, segment p % n_seg), launch head jh (query head h0 + jh * h_step) and
// kept row tau < kept (position (p % n_seg) * w + off + tau * r), the
// -LSE*log2(e) and -Delta of that row, at [(p * n_heads + jh) * Lp + tau];
// padding rows (tau >= kept) get -inf and 0.
__global__ void __launch_bounds__(256) dilated_tables_kernel(const float* __restrict__ lse,
                                                             const float* __restrict__ delta_all,
                                                             float* __restrict__ lse2_t, float* __restrict__ delta_t,
                                                             long long n, int Lp, int kept, int n_heads, int h0,
                                                             int h_step, int n_seg, int w, int off, int r, int S,
                                                             int Hq, int out_h0, int out_hstep) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < n; e += stride) {
    const int tau = static_cast<int>(e % Lp);
    const long long pj = e / Lp;
    const int jh = static_cast<int>(pj % n_heads);
    const long long p = pj / n_heads;
    if (tau >= kept) {
      lse2_t[e] = -INFINITY;
      delta_t[e] = 0.f;
      continue;
    }
    const long long row = ((p / n_seg) * S + (p % n_seg) * w + off + static_cast<long long>(tau) * r) * Hq +
                          out_h0 + (h0 + static_cast<long long>(jh) * h_step) * out_hstep;
    const float l = lse[row];
    lse2_t[e] = l == -INFINITY ? -INFINITY : -l * 1.4426950408889634f;
    delta_t[e] = -delta_all[row];
  }
}

// fp32 -> bf16, n elements (n a multiple of 4, both 16-byte aligned).
__global__ void __launch_bounds__(256) f32_to_bf16_kernel(const float4* __restrict__ x, uint2* __restrict__ y,
                                                          long long n4) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < n4; e += stride) {
    const float4 v = __ldcs(x + e);
    uint2 o;
    o.x = pack_bf16x2(v.x, v.y);
    o.y = pack_bf16x2(v.z, v.w);
    y[e] = o;
  }
}

// Waits on an mbarrier that nothing completes; the bounded wait must give up.
__global__ void wait_selftest_kernel(int* status, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  WaitCtl w{&abort_flag, status, limit_ns};
  if (threadIdx.x == 0) {
    if (!mbar_wait(&bar, 0, w, 0x7E57)) {
      // expected path: the site code is in *status
    }
  }
  __syncthreads();
}

unsigned grid_for(long long units_per_block, long long units) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  long long blocks = (units + units_per_block - 1) / units_per_block;
  const long long cap = static_cast<long long>(sms) * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  return static_cast<unsigned>(blocks);
}

}  // namespace

cudaError_t launch_lse_merge(const float* o_parts, const float* lse_parts, int n_parts, long long rows, int D,
                             void* out, int out_f32, float* lse_out, cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  const unsigned blocks = grid_for(8, rows);
  if (D <= 128 && n_parts == 2) {
    if (out_f32)
      lse_merge_small_kernel<true, 2><<<blocks, 256, 0, stream>>>(o_parts, lse_parts, rows, D, out, lse_out);
    else
      lse_merge_small_kernel<false, 2><<<blocks, 256, 0, stream>>>(o_parts, lse_parts, rows, D, out, lse_out);
  } else if (D <= 128 && n_parts == 1) {
    if (out_f32)
      lse_merge_small_kernel<true, 1><<<blocks, 256, 0, stream>>>(o_parts, lse_parts, rows, D, out, lse_out);
    else
      lse_merge_small_kernel<false, 1><<<blocks, 256, 0, stream>>>(o_parts, lse_parts, rows, D, out, lse_out);
  } else if (out_f32) {
    lse_merge_kernel<true><<<blocks, 256, 0, stream>>>(o_parts, lse_parts, n_parts, rows, D, out, lse_out);
  } else {
    lse_merge_kernel<false><<<blocks, 256, 0, stream>>>(o_parts, lse_parts, n_parts, rows, D, out, lse_out);
  }
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_bwd_preprocess(const void* out, const void* dO, float* delta, long long rows, int D,
                                  cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  bwd_preprocess_kernel<<<grid_for(256, rows), 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(out),
                                                               static_cast<const __nv_bfloat16*>(dO), delta,
                                                               rows, D);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_bwd_prep_rows(const void* out, const void* dO, const float* lse, float* delta_t, float* lse2_t,
                                 int n_rb, int L, int Hl, int D, int Lp, cudaStream_t stream) {
  const long long rows = static_cast<long long>(n_rb) * L * Hl;
  if (rows == 0) return cudaSuccess;
  bwd_prep_rows_kernel<<<grid_for(256, rows), 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(out),
                                                              static_cast<const __nv_bfloat16*>(dO), lse, delta_t,
                                                              lse2_t, rows, L, Hl, D, Lp);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_fill_running(float* o, float* lse, long long rows, int D, cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  const long long n4 = rows * D / 4;
  fill_running_kernel<<<grid_for(256 * 4, n4), 256, 0, stream>>>(reinterpret_cast<float4*>(o), lse, n4, rows);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_dilated_tables(const float* lse, const float* delta_all, float* lse2_t, float* delta_t,
                                  const FwdSub& sb, int Lp, cudaStream_t stream) {
  const long long n = static_cast<long long>(sb.n_prob) * sb.n_heads * Lp;
  if (n == 0) return cudaSuccess;
  dilated_tables_kernel<<<grid_for(256, n), 256, 0, stream>>>(lse, delta_all, lse2_t, delta_t, n, Lp, sb.Lq,
                                                              sb.n_heads, sb.h0, sb.h_step, sb.n_seg, sb.w, sb.off,
                                                              sb.r, sb.S, sb.Hq, sb.out_h0, sb.out_hstep);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_f32_to_bf16(const float* x, void* y, long long n, cudaStream_t stream) {
  if (n == 0) return cudaSuccess;
  const long long n4 = n / 4;
  f32_to_bf16_kernel<<<grid_for(256, n4), 256, 0, stream>>>(reinterpret_cast<const float4*>(x),
                                                            static_cast<uint2*>(y), n4);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_wait_selftest(int* status, unsigned long long limit_ns, cudaStream_t stream) {
  wait_selftest_kernel<<<1, 32, 0, stream>>>(status, limit_ns);
  note_launch();
  return cudaGetLastError();
}

}  // namespace usp
