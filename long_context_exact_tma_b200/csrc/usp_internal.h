// usp_internal.h -- launch interfaces shared by the .cu files of libusp.so.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace usp {

constexpr int kStatusBytes = 256;  // workspace header: device status word + padding

// Sets the calling thread's usp_last_error() message; returns `code`.
int record_error(int code, const char* fmt, ...);

// Layout maps of the gather kernel (see usp_layout.cu).
enum LayoutMap { kZigzagShard = 0, kZigzagUnshard = 1, kSeq2Head = 2, kHead2Seq = 3 };

struct LayoutArgs {
  const uint8_t* src;
  uint8_t* dst;
  int map;
  uint32_t B, S, H, P_u, P_r;  // tokens, heads, mesh
  uint32_t row_bytes;          // bytes of one head row (D * element size)
};
cudaError_t launch_layout(const LayoutArgs& a, cudaStream_t stream);

cudaError_t launch_lse_merge(const float* o_parts, const float* lse_parts, int n_parts, long long rows, int D,
                             void* out, int out_f32, float* lse_out, cudaStream_t stream);
cudaError_t launch_bwd_preprocess(const void* out, const void* dO, float* delta, long long rows, int D,
                                  cudaStream_t stream);
cudaError_t launch_wait_selftest(int* status, unsigned long long limit_ns, cudaStream_t stream);

// Geometry of one attention problem in the head-sharded layout.
struct AttnGeom {
  int B, S, Hq, Hkv, D, causal, P_u, P_r;
  int P, c, L, Hq_l, Hkv_l, G;  // derived
  int n_ranks;                  // P_r * P_u head-sharded ranks
};

struct FwdLaunch {
  AttnGeom g;
  CUtensorMap tm_q, tm_k, tm_v;
  void* out;          // bf16 head-sharded (fused mode)
  float* lse;         // fp32 [ranks][B][L][Hq_l] (fused mode)
  float* o_part;      // fp32 partial O of one ring step (stepwise mode)
  float* lse_part;    // fp32 partial LSE of one ring step (stepwise mode)
  int step;           // ring step (stepwise) or -1 (fused)
  int* status;
  unsigned long long wait_ns;
};
cudaError_t launch_attn_fwd(const FwdLaunch& a, cudaStream_t stream);

// Backward preprocess into the per-head layout the backward kernel streams:
// delta_t/lse2_t [n_ranks*B*Hq_l][Lp] (Lp = L rounded up to 128), holding -Delta
// and -LSE*log2(e); padding rows hold 0 and -inf.
cudaError_t launch_bwd_prep_rows(const void* out, const void* dO, const float* lse, float* delta_t, float* lse2_t,
                                 int n_rb, int L, int Hl, int D, int Lp, cudaStream_t stream);

struct BwdLaunch {
  AttnGeom g;
  CUtensorMap tm_q, tm_k, tm_v, tm_do;
  const float* lse2;   // [n_ranks*B*Hq_l][Lp]: -LSE*log2(e), -inf on padding rows
  const float* delta;  // [n_ranks*B*Hq_l][Lp]: -Delta, 0 on padding rows
  int Lp;
  void* dq;            // bf16, q layout (written by the query-major kernel)
  float* dk;           // fp32, k layout
  float* dv;           // fp32, v layout
  int* status;
  unsigned long long wait_ns;
};
cudaError_t launch_attn_bwd(const BwdLaunch& a, cudaStream_t stream);     // dK, dV (key-major)
cudaError_t launch_attn_bwd_dq(const BwdLaunch& a, cudaStream_t stream);  // dQ (query-major)

}  // namespace usp
