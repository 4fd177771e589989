// Host-side parameter blocks and launchers shared by the C-ABI layer and the
// kernel translation units.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace vsa {

struct PoolParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const int32_t* q_bs;   // [nq] or null (all 64)
  const int32_t* kv_bs;  // [nkv] or null
  int groups;            // B * H
  int nq, nkv;
  float* qc;             // [groups, nq, D]
  float* kc;             // [groups, nkv, D]
  float* vc;
  float* qn;             // [groups, nq] largest row L2 norm of the block's 64 rows, or null
  float* kn;             // [groups, nkv] largest row L2 norm of the block's real rows, or null
  int* status;
};

struct CoarseParams {
  const float* qc;
  const float* kc;
  const float* vc;
  int groups, nq, nkv;
  float scale;
  int topk;        // clamped to [1, nkv]
  int idx_stride;
  int32_t* q2k_idx;
  int32_t* q2k_num;
  float* out_c;    // [groups, nq, D]
  // Optional logit bound (qk_bound null: none): per query block
  // bound_scale * qn[a] * (largest kn of the group), an upper bound on
  // scale_log2 * q.k over the block's query rows and the group's key rows.
  const float* qn;
  const float* kn;
  float* qk_bound;  // [groups, nq]
  float bound_scale;
  int* status;     // device status word (wait timeouts)
};

// One launch of the block-sparse kernel.  Work item = (query block a, head h,
// batch b); "group" = b * H + h.  Rows of q/out are addressed as
//   group * q_rows_per_group + q_tok(a) + t
// and rows of k/v as group * kv_rows_per_group + kv_tok(c) + t, where
// q_tok(a) = 64 a unless a varlen table is given.
struct SparseParams {
  __nv_bfloat16* out;
  const __nv_bfloat16* gate;  // [B, gate_seq, H, D] or null
  const float* out_c;         // [groups, nq, D] or null (no combine)
  const int32_t* q2k_idx;     // [groups, nq, idx_stride]
  const int32_t* q2k_num;     // [groups, nq]
  int idx_stride;
  const int32_t* q_bs;        // [nq] sizes or null (64)
  const int32_t* kv_bs;       // [n kv blocks] sizes or null (64)
  const int32_t* q_tok;       // varlen: first token row of each q block, else null
  const int32_t* kv_tok;      // varlen: first token row of each kv block, else null
  const int32_t* q_kv_base;   // varlen: first kv block of the q block's sequence
  const int32_t* q_kv_count;  // varlen: kv blocks of the q block's sequence
  int B, H, nq, nkv;
  long long q_rows_per_group;
  long long kv_rows_per_group;
  int gate_seq;
  float scale_log2;           // softmax scale * log2(e)
  const float* qk_bound;      // [groups, nq] bound on scale_log2 * q.k (CoarseParams), or null
  int varlen;                 // write only real rows
  int* status;
};

int launch_pool(const PoolParams& p, int D, cudaStream_t stream);
int launch_coarse_topk(const CoarseParams& p, int D, cudaStream_t stream);
// q, k, v: base pointers of the row-major [rows, D] bf16 views.
int launch_sparse(const SparseParams& p, const void* q, const void* k, const void* v,
                  long long q_rows_total, long long kv_rows_total, int D, bool combine,
                  bool gated, cudaStream_t stream);
int launch_selftest_umma(int mode, int D, const void* a, const void* b, float* c,
                         cudaStream_t stream);
int launch_selftest_exp2(const float* x, float* y, long long n, int* mismatch,
                         cudaStream_t stream);

// varlen / metadata helpers (vsa_varlen.cu)
// Logit bound for the varlen entry (same meaning as CoarseParams::qk_bound):
// block row norms of the packed q and k, then per (head, query block) the
// bound over its sequence's KV blocks.
struct VarlenBoundParams {
  const int32_t* q_tok;       // [nqb] first packed row of each query block
  const int32_t* kv_tok;      // [nkvb]
  const int32_t* kv_len;      // [nkvb] real rows
  const int32_t* q_kv_base;   // [nqb] first KV block of the query block's sequence
  const int32_t* q_kv_count;  // [nqb]
  int H, nqb, nkvb;
  long long total_q, total_kv;  // packed rows per head
  float bound_scale;
  float* qn;                  // [H, nqb]
  float* kn;                  // [H, nkvb]
  float* qk_bound;            // [H, nqb]
};
int launch_varlen_bound(const void* q, const void* k, const VarlenBoundParams& p, int D,
                        cudaStream_t stream);
int launch_varlen_aux(const int32_t* blk_tok, const int32_t* blk_len, int n_blocks,
                      int64_t* pack_index, cudaStream_t stream);
int launch_rebase(const int32_t* q2k_idx, const int32_t* q2k_num, const int32_t* q_kv_base,
                  const int32_t* q_kv_count, int H, int nq, int idx_stride, int32_t* out,
                  int* status, cudaStream_t stream);
int launch_gather_tokens(const void* src, void* dst, const int64_t* slot_token, int64_t n_tokens,
                         int64_t n_slots, int64_t groups, int D, bool scatter,
                         cudaStream_t stream);

// cuTensorMapEncodeTiled from the driver (through the runtime's entry-point
// query, so no link against libcuda); null if unavailable.
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn get_encode_fn();

// Device status word of the current device (address via cudaGetSymbolAddress).
int* device_status_ptr();

constexpr float kLog2e = 1.4426950408889634f;

// Softmax scale: the given one, or 1/sqrt(D) when it is <= 0.
float resolve_scale(float scale, int D);

// Arguments of the whole forward (vsa_forward and vsa_forward_noalloc share
// the checks and the launch sequence; only the source of the scratch differs).
struct ForwardArgs {
  const void* q;
  const void* k;
  const void* v;
  const void* gate;
  const int32_t* q_block_sizes;
  const int32_t* kv_block_sizes;
  int B, H, Sq_pad, Skv_pad, D, topk;
  float scale;
  void* out;
  int32_t* q2k_idx;
  int32_t* q2k_num;
  int idx_stride;
  float* out_c;
};
// Host checks of vsa_forward's arguments (everything but the workspace).
int check_forward_args(const ForwardArgs& a);
// Pool, coarse + top-k and the sparse kernel with the fused combine, on
// `stream`, with scratch of vsa_forward_workspace_size bytes at `scratch`.
// `profile`: record the profiling events when the hook is set.
int launch_forward(const ForwardArgs& a, void* scratch, bool profile, cudaStream_t stream);

}  // namespace vsa
