/*
 * usp.h -- C ABI of libusp.so: the per-rank hot path of USP (Ulysses + Ring)
 * context-parallel attention on one NVIDIA B200 (sm_100a), with the P virtual
 * ranks of a P_ulysses x P_ring mesh emulated on the one GPU.
 *
 * Sources (the pages on long_context_exact_tma):
 *   - "Boosting Spec Eagle: USP for Long-Context Training": section "The
 *     Solution" (Ulysses, Ring Attention, their USP hybrid; each ring device
 *     holds a slice of the sequence and exchanges with its neighbours) and
 *     "Implementation Details" (load balancing across the ring).
 *   - DeepSpeed-Ulysses summary, section "Wie DeepSpeed-Ulysses funktioniert":
 *     the input is split along the sequence; an all-to-all before attention
 *     gives each GPU the whole sequence for a subset of heads; afterwards the
 *     results are gathered and re-laid out.
 *   - Blockwise Parallel Transformer (related-papers list of the LSS
 *     Transformer page): attention computed block by block.
 *   - LongNet slides, "Results": attention variants built on FlashAttention,
 *     i.e. exact softmax attention evaluated tile by tile.
 *
 * Notation. P = P_u * P_r ranks; rank r = i * P_u + u (i: ring index, u:
 * Ulysses index). c = S / (2P) tokens per zigzag chunk; rank r holds chunks r
 * and 2P-1-r of the sequence. L = S / P_r tokens per head-sharded rank.
 *
 * Layouts (all row-major, last index contiguous):
 *   global        [B][S][H][D]
 *   rank-major    [P][B][2c][H][D]            (after the zigzag shard)
 *   head-sharded  [P_r][P_u][B][L][H/P_u][D]  (after the seq->head all-to-all;
 *                 the L tokens of rank (i,u) are, for u' = 0..P_u-1 in order,
 *                 the 2c tokens of rank (i,u'))
 *   LSE           head-sharded with D = 1: [P_r][P_u][B][L][Hq/P_u], fp32,
 *                 natural log (global form [B][S][Hq]).
 *
 * Conventions for every call:
 *   - Tensor pointers are DEVICE pointers owned by the caller, 16-byte aligned.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).
 *   - Arguments are validated synchronously; on a bad argument nothing is
 *     launched and a negative usp_status is returned (usp_last_error() then
 *     holds a message). Work is enqueued asynchronously on `stream`.
 *   - The library allocates no device memory: scratch comes from the caller's
 *     workspace (usp_attn_workspace_size). The first 256 bytes of a workspace
 *     hold a device status word that the attention kernels set when a bounded
 *     wait gives up; usp_workspace_status() reads and clears it.
 *   - Supported: D in {64, 128}; Hq % Hkv == 0; Hq % P_u == 0; Hkv % P_u == 0;
 *     S % (2P) == 0. Other shapes return USP_ERR_UNSUPPORTED.
 */
#ifndef USP_H
#define USP_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  USP_OK = 0,
  USP_ERR_INVALID_ARG = -1, /* null/misaligned pointer, negative size, bad enum */
  USP_ERR_UNSUPPORTED = -2, /* a shape outside the supported set */
  USP_ERR_CUDA = -3,        /* a CUDA runtime/driver call failed */
  USP_ERR_TIMEOUT = -4,     /* a kernel's bounded wait gave up; outputs undefined */
  USP_ERR_WORKSPACE = -5    /* workspace missing or smaller than required */
} usp_status;

typedef enum { USP_BF16 = 0, USP_F32 = 1 } usp_dtype;

enum { USP_MODE_FUSED = 0, USP_MODE_STEPWISE = 1 };

/* Library version (major*10000 + minor*100 + patch). */
int usp_version(void);

/* Message for the last non-OK status returned on this thread ("" if none). */
const char* usp_last_error(void);

/* Number of kernels this library has launched in this process (all threads,
 * all devices): a counter for measurement, incremented at every launch. */
unsigned long long usp_launch_count(void);

/*
 * Zigzag shard: global [B][S][H][D] -> rank-major [P][B][2c][H][D]; rank r
 * receives chunks r and 2P-1-r (load balancing of the causal ring, "Boosting
 * Spec Eagle", "Implementation Details"). A bit-exact copy of H*D-element token
 * rows. usp_zigzag_unshard is its inverse. dtype selects 2- or 4-byte
 * elements; D*elem_size must be a multiple of 4 bytes.
 */
int usp_zigzag_shard(const void* src, void* dst, int B, int S, int H, int D, int dtype, int P_u, int P_r,
                     void* stream);
int usp_zigzag_unshard(const void* src, void* dst, int B, int S, int H, int D, int dtype, int P_u, int P_r,
                       void* stream);

/*
 * Ulysses all-to-all emulated as an on-device gather (DeepSpeed-Ulysses,
 * "Wie DeepSpeed-Ulysses funktioniert"): rank-major [P][B][2c][H][D] ->
 * head-sharded [P_r][P_u][B][L][H/P_u][D]. Rank (i,u) receives head group u of
 * every rank (i,u') of its Ulysses group. usp_head2seq_permute is the inverse
 * (the regather after attention). Bit-exact; 16-byte vector copies when the
 * row of H/P_u heads is a multiple of 16 bytes. D may be 1 (the LSE layout).
 */
int usp_seq2head_permute(const void* src, void* dst, int B, int S, int H, int D, int dtype, int P_u, int P_r,
                         void* stream);
int usp_head2seq_permute(const void* src, void* dst, int B, int S, int H, int D, int dtype, int P_u, int P_r,
                         void* stream);

/*
 * Several layout gathers of one map and mesh in ONE launch, e.g. the seq->head
 * all-to-all of Q, K and V before the attention, or the head->seq regather of
 * dQ, dK and dV after it (DeepSpeed-Ulysses summary, "Wie DeepSpeed-Ulysses
 * funktioniert"). Each job is a tensor with its own head count, head-row
 * length and element type, moved exactly as the single call of that map would
 * move it (bit-exact); the launch and its tail are paid once for all of them.
 *   map     USP_MAP_ZIGZAG_SHARD, USP_MAP_ZIGZAG_UNSHARD, USP_MAP_SEQ2HEAD or
 *           USP_MAP_HEAD2SEQ (the layouts of usp_zigzag_shard, usp_zigzag_unshard,
 *           usp_seq2head_permute, usp_head2seq_permute)
 *   jobs    HOST array of n_jobs (1 .. USP_MAX_PERMUTE_JOBS) descriptors; each
 *           job is checked as the single call would check it. Destinations must
 *           not overlap any source or each other.
 */
enum { USP_MAP_ZIGZAG_SHARD = 0, USP_MAP_ZIGZAG_UNSHARD = 1, USP_MAP_SEQ2HEAD = 2, USP_MAP_HEAD2SEQ = 3 };
#define USP_MAX_PERMUTE_JOBS 4
typedef struct {
  const void* src; /* device pointer, 16-byte aligned */
  void* dst;       /* device pointer, 16-byte aligned */
  int H;           /* heads of this tensor */
  int D;           /* elements per head row (1 for an LSE tensor) */
  int dtype;       /* USP_BF16 or USP_F32 */
} usp_permute_job;
int usp_permute_batch(int map, const usp_permute_job* jobs, int n_jobs, int B, int S, int P_u, int P_r,
                      void* stream);

/*
 * Bytes of workspace needed by usp_attn_fwd (bwd = 0, by mode) or
 * usp_attn_bwd (bwd = 1). Returns 0 for an unsupported shape.
 *   fused fwd   : 256 (status word)
 *   stepwise fwd: 256 + 2 * B*S*Hq * (4*D + 4)  (two fp32 partials: the running
 *                 merge of the ring steps done so far and the current step's)
 *   bwd         : 256 + 2 * 4 * B*P_u*P_r*(Hq/P_u)*Lp, Lp = S/P_r rounded up to a
 *                 multiple of 128 (-LSE*log2(e) and -Delta per head and row)
 */
size_t usp_attn_workspace_size(int B, int S, int Hq, int Hkv, int D, int causal, int P_u, int P_r, int mode,
                               int bwd);

/*
 * Forward of exact softmax attention for every virtual rank, block by block
 * over the ring's KV chunks (Ring Attention, "Boosting Spec Eagle", "The
 * Solution"; blockwise attention, BPT), with the partial (O, LSE) pairs of the
 * ring steps combined by log-sum-exp.
 *   q            [P_r][P_u][B][L][Hq/P_u][D]  bf16 (head-sharded)
 *   k, v         [P_r][P_u][B][L][Hkv/P_u][D] bf16
 *   out          like q, bf16: O_i = sum_j softmax_j(scale * q_i.k_j) v_j
 *   lse          [P_r][P_u][B][L][Hq/P_u] fp32, natural log
 * Query head h of rank (i,u) attends kv head h / (Hq/Hkv) of the same rank
 * group u; rank (i,u) at ring step t reads the KV of rank ((i-t) mod P_r, u).
 * causal: key visible iff its original token position <= the query's.
 * scale = 1/sqrt(D).
 * mode USP_MODE_FUSED: one launch, ring steps merged online in the kernel.
 * mode USP_MODE_STEPWISE: the ring algorithm step for step. Each ring step is
 * one launch that writes its fp32 partial (O_t, LSE_t) into the workspace, and
 * the log-sum-exp merge (the kernel of usp_lse_merge) folds it into a running
 * fp32 (O, LSE): two partials in, one out per step, so the workspace holds two
 * partials whatever P_r is. The last step's merge writes out and lse. On return
 * the workspace holds, after the 256-byte status header, o_parts [2][rows][D]
 * and lse_parts [2][rows] (rows = B*S*Hq in the head-sharded row order): slot 0
 * the merge of steps 0..P_r-2, slot 1 the partial of step P_r-1 (for P_r = 1,
 * slot 0 is step 0's partial and slot 1 is unused).
 */
int usp_attn_fwd(const void* q, const void* k, const void* v, void* out, float* lse, int B, int S, int Hq,
                 int Hkv, int D, int causal, int P_u, int P_r, int mode, void* workspace, size_t ws_bytes,
                 void* stream);

/*
 * Backward of usp_attn_fwd for every virtual rank. P is recomputed from the
 * final merged LSE: P_ij = exp(scale q_i.k_j - LSE_i), dP = dO V^T,
 * dS = P o (dP - Delta), Delta_i = sum_d dO_id O_id; dQ = scale dS K,
 * dK = scale dS^T Q, dV = P^T dO, dK/dV summed over the q-heads of a GQA group.
 *   q, out, dO   head-sharded bf16 (out is the forward output)
 *   lse          the forward LSE
 *   dQ           head-sharded bf16 (accumulated in fp32 in TMEM by a query-major
 *                kernel; dK/dV come from a key-major kernel)
 *   dK, dV       head-sharded fp32, [P_r][P_u][B][L][Hkv/P_u][D]
 */
int usp_attn_bwd(const void* q, const void* k, const void* v, const void* out, const float* lse, const void* dO,
                 void* dQ, float* dK, float* dV, int B, int S, int Hq, int Hkv, int D, int causal, int P_u,
                 int P_r, void* workspace, size_t ws_bytes, void* stream);

/*
 * The three phases of usp_attn_bwd, callable on their own (same arguments and
 * layouts; the workspace is the one usp_attn_bwd takes):
 *   usp_attn_bwd_prepare  clears the status word and fills the workspace with
 *                         -Delta_i = -sum_d dO_id O_id and -LSE_i*log2(e) per head
 *                         (padding rows: 0 and -inf);
 *   usp_attn_bwd_dkdv     key-major kernel: dK = scale dS^T Q, dV = P^T dO, summed
 *                         over the GQA group and every ring rank's queries;
 *   usp_attn_bwd_dq       query-major kernel: dQ = scale dS K over every ring step,
 *                         accumulated on chip and written once as bf16.
 * dkdv and dq read only the prepared workspace and the inputs, so they may run in
 * either order (or on two streams) after prepare.
 * usp_attn_bwd_dkdv_bf16 is usp_attn_bwd_dkdv with dK and dV returned in the
 * inputs' type, as dQ is: head-sharded bf16 [P_r][P_u][B][L][Hkv/P_u][D], each
 * element the fp32 sum of usp_attn_bwd_dkdv rounded once to bf16 (nearest even).
 */
int usp_attn_bwd_prepare(const void* out, const float* lse, const void* dO, int B, int S, int Hq, int Hkv, int D,
                         int causal, int P_u, int P_r, void* workspace, size_t ws_bytes, void* stream);
int usp_attn_bwd_dkdv(const void* q, const void* k, const void* v, const void* dO, float* dK, float* dV, int B,
                      int S, int Hq, int Hkv, int D, int causal, int P_u, int P_r, void* workspace, size_t ws_bytes,
                      void* stream);
int usp_attn_bwd_dq(const void* q, const void* k, const void* v, const void* dO, void* dQ, int B, int S, int Hq,
                    int Hkv, int D, int causal, int P_u, int P_r, void* workspace, size_t ws_bytes, void* stream);
int usp_attn_bwd_dkdv_bf16(const void* q, const void* k, const void* v, const void* dO, void* dK, void* dV, int B,
                           int S, int Hq, int Hkv, int D, int causal, int P_u, int P_r, void* workspace,
                           size_t ws_bytes, void* stream);

/*
 * Sparse and variable-length attention under the Ulysses layout
 * (DeepSpeed-Ulysses summary, "Hauptmerkmale von DeepSpeed-Ulysses", item 3:
 * dense and sparse attention alike -- after the all-to-all each rank holds
 * whole sequences for its heads, so an attention pattern applies unchanged).
 * usp_attn_fwd_masked / usp_attn_bwd_masked are usp_attn_fwd (fused mode) and
 * usp_attn_bwd with a visibility mask on top of causality, both in ORIGINAL
 * token positions (the zigzag and the all-to-all are undone by the kernels):
 *   block_mask  DEVICE bytes [B][Hq][S/128][S/128] (global query head index):
 *               key block kb is visible to query block qb iff
 *               block_mask[b][h][qb][kb] != 0; blocks are 128 positions, the
 *               kernels' tile, so masked-off blocks are skipped whole; or NULL.
 *   cu_seqlens  DEVICE int32 [n_docs + 1]: packed variable-length sequences
 *               (documents [cu[d], cu[d+1]), non-decreasing, cu[0] = 0,
 *               cu[n_docs] = S, shared by the batch); a query sees only keys of
 *               its own document; or NULL. Other values give undefined results
 *               but never an access outside cu[0 .. n_docs].
 * A query row with no visible key gets O = 0 and LSE = -inf and contributes no
 * gradient. Masks need zigzag chunks that are whole tiles: S / (2 P_u P_r) a
 * multiple of 128 (else USP_ERR_UNSUPPORTED). Workspaces are those of
 * usp_attn_fwd (fused) and usp_attn_bwd. A NULL mask, or one with both
 * pointers NULL, is the unmasked call.
 */
typedef struct {
  const unsigned char* block_mask;
  const int* cu_seqlens;
  int n_docs;
} usp_attn_mask;
int usp_attn_fwd_masked(const void* q, const void* k, const void* v, void* out, float* lse, int B, int S, int Hq,
                        int Hkv, int D, int causal, int P_u, int P_r, const usp_attn_mask* mask, void* workspace,
                        size_t ws_bytes, void* stream);
int usp_attn_bwd_masked(const void* q, const void* k, const void* v, const void* out, const float* lse,
                        const void* dO, void* dQ, float* dK, float* dV, int B, int S, int Hq, int Hkv, int D,
                        int causal, int P_u, int P_r, const usp_attn_mask* mask, void* workspace, size_t ws_bytes,
                        void* stream);

/*
 * The per-rank compute of a REAL multi-GPU USP mesh: one process per GPU holds
 * one rank r = i * P_u + u and calls these between its own NCCL collectives
 * ("Boosting Spec Eagle", "The Solution": ring devices hold slices of the
 * sequence and pass key/value blocks to their neighbours; DeepSpeed-Ulysses
 * summary, "Wie DeepSpeed-Ulysses funktioniert": all-to-all before and after
 * attention). Shapes (B, S, Hq, Hkv, D, causal, P_u, P_r) are the GLOBAL ones
 * of the mesh, as for usp_attn_fwd; the buffers are the rank's own:
 *   rank-local tokens  [B][T][H][D], T = S / (P_u P_r) (zigzag chunks r, 2P-1-r)
 *   head-sharded       [B][L][H/P_u][D], L = S / P_r (the slice [i][u] of the
 *                      one-GPU head-sharded layout)
 *
 * usp_ulysses_pack: the local halves of the Ulysses all-to-all among the G =
 * P_u ranks of a group (jobs as for usp_permute_batch, H = the tensor's total
 * heads, a multiple of G; T tokens per rank):
 *   USP_MAP_PACK_HEADS    [B][T][H][D] -> [G][B][T][H/G][D]  send buffer, seq->head
 *   USP_MAP_UNPACK_TOKENS [G][B][T][H/G][D] -> [B][G*T][H/G][D] received, seq->head
 *   USP_MAP_PACK_TOKENS   [B][G*T][H/G][D] -> [G][B][T][H/G][D] send buffer, head->seq
 *   USP_MAP_UNPACK_HEADS  [G][B][T][H/G][D] -> [B][T][H][D]  received, head->seq
 * with an equal-split all-to-all over the group between pack and unpack.
 *
 * usp_ring_fwd_step: ring step t of rank (i, u): its head-sharded q against the
 * KV block of ring rank j = (i - t) mod P_r (same u) that it holds now; writes
 * the step's fp32 partial o_part [B][L][Hq/P_u][D] and lse_part [B][L][Hq/P_u]
 * (rows that see no key of the block: LSE = -inf, O = 0). Fold the partials
 * with usp_lse_merge (in place into a running fp32 result). Workspace 256 B.
 *
 * usp_ring_fwd_accumulate: the same step, folded into a running fp32 result
 * instead: step t = 0 writes o_run / lse_run ([B][L][Hq/P_u][D], [B][L][Hq/P_u])
 * like usp_ring_fwd_step; every later step merges its partial into them by the
 * log-sum-exp merge in the kernel's epilogue (one buffer, no merge launch).
 * Call it for t = 0, 1, ... in order; usp_lse_merge with n_parts = 1 then
 * writes the bf16 O and the LSE.
 *
 * usp_ring_bwd_prepare: the per-head -LSE*log2(e) and -Delta tables of the
 * rank's rows from its final out, lse and dO (workspace of
 * usp_ring_workspace_size(..., bwd = 1)).
 * usp_ring_bwd_step: ring step t: ADDS this rank's contribution to the
 * gradients of the block it holds, dk_acc / dv_acc (fp32, the gradients
 * travelling with the block), and to its own dq_acc (fp32); when dq_out (bf16,
 * may be NULL) is given, the final dQ = dq_acc + this step is written there
 * instead of into dq_acc (call it so on the last step).
 */
#define USP_MAP_PACK_HEADS 4
#define USP_MAP_UNPACK_TOKENS 5
#define USP_MAP_PACK_TOKENS 6
#define USP_MAP_UNPACK_HEADS 7
int usp_ulysses_pack(int map, const usp_permute_job* jobs, int n_jobs, int B, int T, int G, void* stream);
size_t usp_ring_workspace_size(int B, int S, int Hq, int Hkv, int D, int causal, int P_u, int P_r, int bwd);
int usp_ring_fwd_step(const void* q, const void* k, const void* v, float* o_part, float* lse_part, int B, int S,
                      int Hq, int Hkv, int D, int causal, int P_u, int P_r, int i, int u, int t, void* workspace,
                      size_t ws_bytes, void* stream);
int usp_ring_fwd_accumulate(const void* q, const void* k, const void* v, float* o_run, float* lse_run, int B, int S,
                            int Hq, int Hkv, int D, int causal, int P_u, int P_r, int i, int u, int t,
                            void* workspace, size_t ws_bytes, void* stream);
int usp_ring_bwd_prepare(const void* out, const float* lse, const void* dO, int B, int S, int Hq, int Hkv, int D,
                         int causal, int P_u, int P_r, void* workspace, size_t ws_bytes, void* stream);
int usp_ring_bwd_step(const void* q, const void* k, const void* v, const void* dO, float* dq_acc, void* dq_out,
                      float* dk_acc, float* dv_acc, int B, int S, int Hq, int Hkv, int D, int causal, int P_u, int P_r,
                      int i, int u, int t, void* workspace, size_t ws_bytes, void* stream);

/*
 * Bytes of the static device scratch behind usp_attn_bwd_noalloc (32 MiB).
 */
#define USP_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)

/*
 * usp_attn_bwd without a workspace argument. The paper has no counterpart:
 * this is a convenience of this library for callers that cannot allocate
 * device memory for a workspace, such as code running while a framework's
 * caching allocator or a pool reserved at start-up owns the device memory
 * (a cudaMalloc behind its back can fail or fragment it), or serving loops
 * that must not allocate after initialisation (cudaMalloc can synchronise the
 * device).
 *
 * Arguments and results are those of usp_attn_bwd. The scratch is a
 * file-scope static __device__ array of USP_NOALLOC_SCRATCH_BYTES bytes, which
 * every GPU that loads this part of the library holds until the process exits.
 * It has the layout of the usp_attn_bwd workspace: the 256-byte status header,
 * then the per-head -LSE*log2(e) and -Delta tables. Each call clears the status
 * word; the two tables are rewritten in full (padding rows included) by the
 * prepare step of every call, so nothing else has to start at zero. A problem
 * whose usp_attn_workspace_size(..., bwd=1) exceeds that size is rejected with
 * USP_ERR_WORKSPACE before anything is launched. The call allocates nothing:
 * no cudaMalloc, no cudaFree, no allocating library routine.
 *
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress, which may load the library's device code) and keeps
 * it for the life of the process; make that first call before any stream
 * capture, and do not use this entry point across a cudaDeviceReset (the
 * device code, and with it the array, may then load at another address).
 * Every call shares the one array; calls whose work overlaps on the GPU (other
 * streams, other threads) race on it and must be serialised by the caller. A
 * bounded device wait that gives up during a call records its site in the
 * array's status word; usp_attn_bwd_noalloc_status reads it.
 */
int usp_attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* out, const float* lse,
                         const void* dO, void* dQ, float* dK, float* dV, int B, int S, int Hq, int Hkv, int D,
                         int causal, int P_u, int P_r, void* stream);

/*
 * LongNet dilated attention, forward (LongNet slides, "Abstract": dilated
 * attention is a drop-in replacement for standard attention; "Results":
 * segment lengths w = {2048, ..., 32768} with dilation ratios r = {1, 2, 4, 6,
 * 12}). For each of the n_pairs pairs (w[p], r[p]):
 *   - the sequence is cut into segments of w[p] tokens;
 *   - in every segment, every r[p]-th row is kept, starting at the offset
 *     h mod r[p] of query head h (the kv head h / (Hq/Hkv) uses the same rows);
 *   - exact softmax attention runs among the kept rows of each segment
 *     (causal: key position <= query position);
 * and the pairs' results are combined with weights proportional to their
 * softmax denominators: O = sum_p Z_p O_p / sum_p Z_p, LSE = log sum_p Z_p,
 * i.e. the log-sum-exp merge. A row that no pair keeps gets O = 0, LSE = -inf.
 *   q            [B][S][Hq][D]  bf16 (global layout; one device's sequence)
 *   k, v         [B][S][Hkv][D] bf16
 *   out          [B][S][Hq][D]  bf16;  lse [B][S][Hq] fp32, natural log
 *   w, r         HOST arrays of n_pairs (1 .. USP_DILATED_MAX_PAIRS) ints;
 *                S % w[p] == 0 and 1 <= r[p] <= w[p]
 *   workspace    usp_dilated_workspace_size(B, S, Hq, D) bytes: the status
 *                header, then the running fp32 O [B*S*Hq][D] and LSE [B*S*Hq]
 * D in {64, 128}. One kernel launch per (pair, head offset), each reading the
 * kept rows straight from q, k, v through strided TMA tensor maps, plus an
 * initialisation and a final merge launch. Scale 1/sqrt(D).
 */
#define USP_DILATED_MAX_PAIRS 16
size_t usp_dilated_workspace_size(int B, int S, int Hq, int D);
/*
 * usp_dilated_attn_bwd: the backward of usp_dilated_attn_fwd. With the final
 * (merged) LSE and Delta_i = dO_i . O_i, every pair contributes at its kept
 * rows the attention backward of its segments -- P_ij = exp(s_ij - LSE_i),
 * dS_ij = P_ij (dO_i . V_j - Delta_i), dQ = scale dS K, dK = scale dS^T Q,
 * dV = P^T dO -- and the pairs' contributions are summed (a key shown to a
 * query by two pairs counts twice, as in the forward).
 *   out, lse   the forward's outputs;  dO [B][S][Hq][D] bf16
 *   dQ         [B][S][Hq][D] bf16;  dK, dV [B][S][Hkv][D] fp32 (overwritten)
 *   workspace  usp_dilated_bwd_workspace_size(B, S, Hq, D, n_pairs, w, r)
 *              bytes (status, Delta of every row, an fp32 dQ, and one slot of
 *              the row tables of the largest launch per head offset, up to
 *              16: the head offsets of a pair write disjoint rows and run on
 *              up to 16 streams at once, the forward's too); 0 for an
 *              unsupported shape.
 */
size_t usp_dilated_bwd_workspace_size(int B, int S, int Hq, int D, int n_pairs, const int* w, const int* r);
int usp_dilated_attn_bwd(const void* q, const void* k, const void* v, const void* out, const float* lse,
                         const void* dO, void* dQ, float* dK, float* dV, int B, int S, int Hq, int Hkv, int D,
                         int causal, int n_pairs, const int* w, const int* r, void* workspace, size_t ws_bytes,
                         void* stream);
int usp_dilated_attn_fwd(const void* q, const void* k, const void* v, void* out, float* lse, int B, int S, int Hq,
                         int Hkv, int D, int causal, int n_pairs, const int* w, const int* r, void* workspace,
                         size_t ws_bytes, void* stream);

/*
 * usp_rows_copy: up to USP_MAX_ROWS_JOBS affine row copies in one launch, the
 * data movement around the LongNet collectives below (packing the kept rows of
 * a rank before an all-gather, compacting the gathered blocks, and the reverse
 * for the reduce-scatter of their gradients). Job x copies, for b < n_b,
 * k < n_k, j < n_j, one row of D elements
 *   src[b * s_b + (s_k0 + k * s_kstep) * s_k + ((s_h0 + j * s_hstep) / s_hdiv) * s_h]
 *   -> dst[b * d_b + (d_k0 + k * d_kstep) * d_k + ((d_h0 + j * d_hstep) / d_hdiv) * d_h]
 * (strides in elements), assigning, or adding when `add` (USP_F32 only; the
 * rows of one (b, k) are added in j order, so several j may share a
 * destination row). dtype USP_BF16 or USP_F32 for both sides; D * element size
 * a multiple of 16 bytes and every row 16-byte aligned. Different jobs of one
 * call must not write the same destination row. USP_ERR_INVALID_ARG otherwise.
 */
#define USP_MAX_ROWS_JOBS 16
typedef struct {
  const void* src;
  void* dst;
  int dtype;
  int add;
  int n_b, n_k, n_j, D;
  long long s_b, s_k, s_h;
  int s_k0, s_kstep, s_h0, s_hstep, s_hdiv;
  long long d_b, d_k, d_h;
  int d_k0, d_kstep, d_h0, d_hstep, d_hdiv;
} usp_rows_job;
int usp_rows_copy(const usp_rows_job* jobs, int n_jobs, void* stream);

/*
 * LongNet's distributed layout, per rank (LongNet slides, "LONGNET as a
 * Distributed Trainer": a segment no longer than a device's slice is computed
 * locally; a longer one has its key/value rows brought together by an
 * all-gather, and the local queries attend those global rows; in the backward
 * the all-gather becomes a reduce-scatter). The sequence of S tokens is split
 * into M contiguous slices of T = S / M tokens, rank d holding positions
 * [d*T, (d+1)*T) of q [B][T][Hq][D], k, v [B][T][Hkv][D] (bf16). Each (w, r)
 * pair of usp_dilated_attn_fwd is then either
 *   local     w <= T (T % w == 0): usp_longnet_fwd_local / _bwd_local, the
 *             dilated attention of the rank's own segments;
 *   gathered  w > T (w % T == 0): the segment spans G = w / T ranks; the rank
 *             is number g = d mod G in it. For every head offset o < min(r, Hq)
 *             the query heads o, o + r, ... (n_sel of them) keep the segment
 *             rows at positions = o (mod r). usp_longnet_rows gives this rank's
 *             share of those rows: the first kept local row lp0, its index k_lo
 *             among the segment's kept rows, their count n_rows (local rows
 *             lp0, lp0 + r, ...), and the segment's total n_kept. The caller
 *             packs the rank's kept K/V rows of the kv heads of those query
 *             heads (usp_rows_copy), all-gathers them over the segment's G
 *             ranks, compacts them in kept order into kc, vc
 *             [B][n_kept][n_sel][D] bf16 (head j = the kv head of query head
 *             o + j r) and calls usp_longnet_fwd_cross: the rank's n_rows
 *             kept query rows (kept indices k_lo ...) against all n_kept rows,
 *             causal by kept index.
 * Every call folds into a running fp32 (O, LSE) in the workspace
 * (usp_longnet_fwd_begin resets it, usp_longnet_fwd_end writes out [B][T][Hq][D]
 * bf16 and lse [B][T][Hq] fp32 with the pairs combined as in
 * usp_dilated_attn_fwd), so the rank's result equals rows [d*T, (d+1)*T) of
 * usp_dilated_attn_fwd on the whole sequence.
 * Backward: usp_longnet_bwd_begin (Delta of every row; dQ accumulator, dK and
 * dV zeroed) with the final out and lse; per local pair usp_longnet_bwd_local
 * (adds to dK, dV [B][T][Hkv][D] fp32); per gathered (pair, offset)
 * usp_longnet_bwd_cross with the same kc, vc: writes this rank's queries'
 * contribution to the gathered rows' gradients dkc, dvc [B][n_kept][n_sel][D]
 * fp32 (overwritten), which the caller reduce-scatters over the segment and
 * adds at its own kept rows (usp_rows_copy with add); usp_longnet_bwd_end
 * writes dQ [B][T][Hq][D] bf16.
 * Concurrency: the offsets of one gathered pair write disjoint heads (and,
 * backward, their own dkc/dvc and the row-table slot o mod 16 of the
 * workspace), so their usp_longnet_fwd_cross / usp_longnet_bwd_cross calls may
 * run on different streams at the same time, as long as offsets that share a
 * slot (o mod 16) share a stream; calls of different pairs, and the local
 * calls, must not overlap each other.
 * Workspace: usp_longnet_workspace_size(B, T, Hq, D, n_pairs, w, r, bwd) for
 * the pairs that will be passed (0 for an unsupported shape). D in {64, 128},
 * Hq % Hkv == 0, 1 <= r <= w.
 */
int usp_longnet_rows(int T, int w, int r, int o, int g, int* lp0, int* k_lo, int* n_rows, int* n_kept);
size_t usp_longnet_workspace_size(int B, int T, int Hq, int D, int n_pairs, const int* w, const int* r, int bwd);
int usp_longnet_fwd_begin(int B, int T, int Hq, int D, void* workspace, size_t ws_bytes, void* stream);
int usp_longnet_fwd_local(const void* q, const void* k, const void* v, int B, int T, int Hq, int Hkv, int D,
                          int causal, int w, int r, void* workspace, size_t ws_bytes, void* stream);
int usp_longnet_fwd_cross(const void* q, const void* kc, const void* vc, int B, int T, int Hq, int Hkv, int D,
                          int causal, int w, int r, int o, int g, void* workspace, size_t ws_bytes, void* stream);
int usp_longnet_fwd_end(void* out, float* lse, int B, int T, int Hq, int D, void* workspace, size_t ws_bytes,
                        void* stream);
int usp_longnet_bwd_begin(const void* out, const float* lse, const void* dO, float* dK, float* dV, int B, int T,
                          int Hq, int Hkv, int D, void* workspace, size_t ws_bytes, void* stream);
int usp_longnet_bwd_local(const void* q, const void* k, const void* v, const void* dO, const float* lse, float* dK,
                          float* dV, int B, int T, int Hq, int Hkv, int D, int causal, int w, int r, void* workspace,
                          size_t ws_bytes, void* stream);
int usp_longnet_bwd_cross(const void* q, const void* kc, const void* vc, const void* dO, const float* lse,
                          float* dkc, float* dvc, int B, int T, int Hq, int Hkv, int D, int causal, int w, int r,
                          int o, int g, void* workspace, size_t ws_bytes, void* stream);
int usp_longnet_bwd_end(void* dQ, int B, int T, int Hq, int D, void* workspace, size_t ws_bytes, void* stream);

/*
 * usp_workspace_status for the static scratch of usp_attn_bwd_noalloc (which a
 * caller cannot name): synchronises `stream`, returns USP_ERR_TIMEOUT if a
 * kernel of an earlier usp_attn_bwd_noalloc call on the current device recorded
 * a timed-out wait (and clears the word), USP_OK otherwise; `site` (may be
 * NULL) receives the recorded site code. Allocates nothing.
 */
int usp_attn_bwd_noalloc_status(int* site, void* stream);

/*
 * Log-sum-exp merge of n_parts ring-step partials (the partial results each
 * ring step produces, "Boosting Spec Eagle", "The Solution"):
 *   LSE = m + log sum_t exp(LSE_t - m),  m = max_t LSE_t
 *   O   = sum_t exp(LSE_t - LSE) O_t
 * A partial with LSE_t = -inf (no visible key) contributes nothing; a row with
 * every LSE_t = -inf yields O = 0, LSE = -inf.
 *   o_parts    [n_parts][rows][D] fp32;  lse_parts [n_parts][rows] fp32
 *   out        [rows][D], bf16 or fp32 (out_dtype);  lse_out [rows] fp32
 * D must be a multiple of 4 (<= 256). With out_dtype USP_F32 the merge may run
 * in place: out == o_parts and lse_out == lse_parts (partial 0 is overwritten
 * by the result), which is how the stepwise forward streams its ring merge.
 * Any other overlap of the outputs with the inputs is undefined.
 */
int usp_lse_merge(const float* o_parts, const float* lse_parts, int n_parts, long long rows, int D, void* out,
                  int out_dtype, float* lse_out, void* stream);

/*
 * Backward preprocess: Delta_i = sum_d dO_id * O_id in fp32, for `rows` rows of
 * D bf16 elements (any row-major layout, the same for both inputs).
 */
int usp_bwd_preprocess(const void* out, const void* dO, float* delta, long long rows, int D, void* stream);

/*
 * Synchronises `stream`, returns USP_ERR_TIMEOUT if a kernel that used this
 * workspace recorded a timed-out wait since the last call (and clears the
 * word), USP_OK otherwise. `site` (may be NULL) receives the recorded site code.
 */
int usp_workspace_status(void* workspace, int* site, void* stream);

/*
 * Limit of every bounded device wait launched by this thread from now on, in
 * nanoseconds (default 2e9). A test hook: a very small limit makes waits give up.
 */
void usp_set_wait_limit_ns(unsigned long long ns);

/*
 * Self-test of the bounded-wait machinery: launches one CTA that waits on an
 * mbarrier nothing will ever complete, with limit `limit_ns`; the wait gives up,
 * the kernel records its site and returns. Then usp_workspace_status on the
 * same workspace reports USP_ERR_TIMEOUT.
 */
int usp_selftest_wait_timeout(void* workspace, size_t ws_bytes, unsigned long long limit_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* USP_H */
