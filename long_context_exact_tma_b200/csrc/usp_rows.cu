// usp_rows.cu -- affine row copies (usp_rows_copy): the data movement around
// the all-gather and reduce-scatter of LongNet's distributed layout (LongNet
// slides, "LONGNET as a Distributed Trainer"): a rank's kept key/value rows
// packed before the all-gather, the gathered blocks compacted in kept order,
// and the reverse, with an add, for the gradients after the reduce-scatter.
//
// A job is a 3-D set of rows (b, k, j) of D elements, each read at an affine
// row / floored-affine head index of the source and written (or added) at one
// of the destination. Threads own one 16-byte chunk of one (b, k) row group
// and walk j in order, so rows of one (b, k) that share a destination row (GQA
// heads added into their kv head) never race. HBM-bound: 16-byte loads and
// stores, consecutive threads on consecutive chunks of a row.
#include "../../include/usp.h"
#include "usp_internal.h"

namespace usp {
namespace {

struct RowsBatch {
  usp_rows_job job[USP_MAX_ROWS_JOBS];
  long long start[USP_MAX_ROWS_JOBS + 1];  // first work unit of each job (units = n_b * n_k * chunks)
  int chunks[USP_MAX_ROWS_JOBS];           // 16-byte chunks of a row
  int es[USP_MAX_ROWS_JOBS];               // element size
  int n;
};

__global__ void __launch_bounds__(256) rows_copy_kernel(const __grid_constant__ RowsBatch bt) {
  const long long total = bt.start[bt.n];
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long u = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; u < total; u += stride) {
    int x = 0;
    while (u >= bt.start[x + 1]) ++x;
    const usp_rows_job& J = bt.job[x];
    const long long v = u - bt.start[x];
    const int nc = bt.chunks[x], es = bt.es[x];
    const int c = static_cast<int>(v % nc);
    const long long rg = v / nc;
    const int k = static_cast<int>(rg % J.n_k);
    const long long b = rg / J.n_k;
    const long long srow = b * J.s_b + static_cast<long long>(J.s_k0 + static_cast<long long>(k) * J.s_kstep) * J.s_k;
    const long long drow = b * J.d_b + static_cast<long long>(J.d_k0 + static_cast<long long>(k) * J.d_kstep) * J.d_k;
    const uint8_t* src = static_cast<const uint8_t*>(J.src);
    uint8_t* dst = static_cast<uint8_t*>(J.dst);
    for (int j = 0; j < J.n_j; ++j) {
      const long long sh = static_cast<long long>((J.s_h0 + static_cast<long long>(j) * J.s_hstep) / J.s_hdiv);
      const long long dh = static_cast<long long>((J.d_h0 + static_cast<long long>(j) * J.d_hstep) / J.d_hdiv);
      const uint4* s4 = reinterpret_cast<const uint4*>(src + (srow + sh * J.s_h) * es) + c;
      uint4* d4 = reinterpret_cast<uint4*>(dst + (drow + dh * J.d_h) * es) + c;
      const uint4 val = *s4;
      if (J.add) {
        const uint4 old = *d4;
        uint4 sum;
        sum.x = __float_as_uint(__uint_as_float(old.x) + __uint_as_float(val.x));
        sum.y = __float_as_uint(__uint_as_float(old.y) + __uint_as_float(val.y));
        sum.z = __float_as_uint(__uint_as_float(old.z) + __uint_as_float(val.z));
        sum.w = __float_as_uint(__uint_as_float(old.w) + __uint_as_float(val.w));
        *d4 = sum;
      } else {
        *d4 = val;
      }
    }
  }
}

bool al16(long long x) { return (x & 15) == 0; }

}  // namespace
}  // namespace usp

extern "C" int usp_rows_copy(const usp_rows_job* jobs, int n_jobs, void* stream) {
  using usp::record_error;
  if (!jobs || n_jobs < 1 || n_jobs > USP_MAX_ROWS_JOBS)
    return record_error(USP_ERR_INVALID_ARG, "n_jobs must be 1..%d with a job array", USP_MAX_ROWS_JOBS);
  usp::RowsBatch bt{};
  long long units = 0;
  int n = 0;
  for (int x = 0; x < n_jobs; ++x) {
    const usp_rows_job& J = jobs[x];
    const int es = J.dtype == USP_BF16 ? 2 : J.dtype == USP_F32 ? 4 : 0;
    if (es == 0) return record_error(USP_ERR_INVALID_ARG, "job %d: dtype must be USP_BF16 or USP_F32", x);
    if (J.add && J.dtype != USP_F32) return record_error(USP_ERR_INVALID_ARG, "job %d: add needs USP_F32", x);
    if (J.n_b < 0 || J.n_k < 0 || J.n_j < 0 || J.D <= 0)
      return record_error(USP_ERR_INVALID_ARG, "job %d: negative count or D <= 0", x);
    if (J.s_hdiv < 1 || J.d_hdiv < 1 || J.s_k0 < 0 || J.d_k0 < 0 || J.s_h0 < 0 || J.d_h0 < 0 || J.s_kstep < 0 ||
        J.d_kstep < 0 || J.s_hstep < 0 || J.d_hstep < 0 || J.s_b < 0 || J.s_k < 0 || J.s_h < 0 || J.d_b < 0 ||
        J.d_k < 0 || J.d_h < 0)
      return record_error(USP_ERR_INVALID_ARG, "job %d: negative offset or stride, or a divisor below 1", x);
    if (static_cast<long long>(J.D) * es % 16 != 0)
      return record_error(USP_ERR_INVALID_ARG, "job %d: D * element size must be a multiple of 16 bytes", x);
    if (J.n_b == 0 || J.n_k == 0 || J.n_j == 0) continue;  // nothing to move
    if (!J.src || !J.dst) return record_error(USP_ERR_INVALID_ARG, "job %d: null pointer", x);
    if (!usp::al16(reinterpret_cast<long long>(J.src)) || !usp::al16(reinterpret_cast<long long>(J.dst)) ||
        !usp::al16(J.s_b * es) || !usp::al16(J.s_k * es) || !usp::al16(J.s_h * es) || !usp::al16(J.d_b * es) ||
        !usp::al16(J.d_k * es) || !usp::al16(J.d_h * es))
      return record_error(USP_ERR_INVALID_ARG, "job %d: pointers and strides must keep rows 16-byte aligned", x);
    bt.job[n] = J;
    bt.es[n] = es;
    bt.chunks[n] = J.D * es / 16;
    bt.start[n] = units;
    units += static_cast<long long>(J.n_b) * J.n_k * bt.chunks[n];
    ++n;
  }
  if (n == 0) return USP_OK;
  bt.start[n] = units;
  bt.n = n;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long want = (units + 255) / 256;
  const unsigned grid = static_cast<unsigned>(want < 8LL * sms ? want : 8LL * sms);
  usp::rows_copy_kernel<<<grid, 256, 0, st>>>(bt);
  usp::note_launch();
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? USP_OK : record_error(USP_ERR_CUDA, "rows copy launch: %s", cudaGetErrorString(e));
}
