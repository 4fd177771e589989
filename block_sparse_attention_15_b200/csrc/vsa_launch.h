// Host-side parameter blocks and launchers shared by the C-ABI layer and the
// kernel translation units.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace vsa {

// Element strides of a [batch][head][sequence slot][head dim] view whose head
// dim is contiguous.
struct Strides3 {
  long long b, h, s;
};

// Tensor-map dimension (1..3) that holds each of the sequence, head and
// batch axes of a 4D tile map (dimension 0 is the head dim): the three axes
// are ordered by stride on the host.
struct TmaAxes {
  int s, h, b;
};

struct PoolParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  Strides3 q_st, k_st, v_st;
  const int32_t* q_bs;   // [nq] or null (all 64)
  const int32_t* kv_bs;  // [nkv] or null
  int groups;            // B * H
  int H;
  int block;             // slots per block: 64 or 128
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
// batch b); "group" = b * H + h.  Token t of query block a is sequence slot
// q_tok(a) + t of (b, h) in q and out, token t of KV block c is slot
// kv_tok(c) + t in k and v, where q_tok(a) = 64 a and kv_tok(c) = 64 c unless
// a varlen table is given.  Every tensor is a strided [B, H, S, D] view.
struct SparseParams {
  __nv_bfloat16* out;
  Strides3 out_st;
  const __nv_bfloat16* gate;  // strided [B, H, Sq, D] view or null
  Strides3 gate_st;
  TmaAxes q_ax, k_ax, v_ax;   // filled by launch_sparse
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
  float scale_log2;           // softmax scale * log2(e)
  const float* qk_bound;      // [groups, nq] bound on scale_log2 * q.k (CoarseParams), or null
  float* lse;                 // [groups, lse_seq] natural-log log-sum-exp per query row, or null
  long long lse_seq;
  int varlen;                 // write only real rows
  // 128-slot kernel only: log2 of the 128-slot sub-blocks per caller block
  // (0: blocks of 128; 1: blocks of 256 walked as two 128-row halves, each
  // selected block read as two 128-key sub-tiles)
  int sub;
  int* status;
};

// Host-to-device copy of a small host table through the library's per-device
// page-locked staging ring (capi.cu): asynchronous on `st`; `src` may be
// released as soon as the call returns.
int stage_copy_h2d(void* dst, const void* src, size_t bytes, cudaStream_t st);
int launch_pool(const PoolParams& p, int D, cudaStream_t stream);
int launch_coarse_topk(const CoarseParams& p, int D, cudaStream_t stream);
// q, k, v: strided [B, H, S, D] bf16 views with S = q_seq / kv_seq slots
// (element strides multiples of 8, bases 16-byte aligned).
int launch_sparse(const SparseParams& p, const void* q, Strides3 q_st, long long q_seq,
                  const void* k, Strides3 k_st, const void* v, Strides3 v_st, long long kv_seq,
                  int D, bool combine, bool gated, cudaStream_t stream);
int launch_selftest_umma(int mode, int D, const void* a, const void* b, float* c,
                         cudaStream_t stream);
// The 128-token block path (sparse128_fwd.cu): same parameters, blocks of
// 128 slots, no varlen tables.
int launch_sparse128(const SparseParams& p, const void* q, Strides3 q_st, long long q_seq,
                     const void* k, Strides3 k_st, const void* v, Strides3 v_st, long long kv_seq,
                     int D, bool combine, bool gated, cudaStream_t stream);
int launch_selftest128(int mode, int D, const void* a, const void* b, float* c,
                       cudaStream_t stream);
// 4-D tile map of a strided [B, H, S, D] bf16 view with boxes of 64 head
// dims x box_rows slots (sparse_fwd.cu).
bool make_view_map_rows(CUtensorMap* map, TmaAxes* ax, const void* base, int D, long long S,
                        int H, int B, Strides3 st, int box_rows);
int launch_selftest_exp2(const float* x, float* y, long long n, int* mismatch,
                         cudaStream_t stream);

// Backward of the 64-slot block-sparse attention (sparse_bwd.cu).  Work of
// the dq pass: (query block, head, batch); of the dk/dv pass: (KV block,
// head, batch).  Tables as in SparseParams (null: regular layout).
struct BwdParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const __nv_bfloat16* dout;
  Strides3 q_st, k_st, v_st, do_st;
  TmaAxes q_ax, k_ax, v_ax, do_ax;  // filled by launch_backward
  const float* lse;           // [groups, q_seq] natural-log log-sum-exp
  float* delta;               // [groups, q_seq] scratch: sum_d dout * out
  long long q_seq, kv_seq;
  const int32_t* q2k_idx;     // [groups, nq, idx_stride]
  const int32_t* q2k_num;
  int idx_stride;
  const int32_t* q_bs;
  const int32_t* kv_bs;
  const int32_t* q_tok;
  const int32_t* kv_tok;
  const int32_t* q_kv_base;
  const int32_t* q_kv_count;
  int32_t* k2q;               // [groups, nkv, nq] scratch: query block | multiplicity << 16
  int32_t* k2q_num;           // [groups, nkv]
  __nv_bfloat16* dq;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  Strides3 dq_st, dk_st, dv_st;
  int B, H, nq, nkv;
  float scale, scale_log2;
  int varlen;
  int* status;
};
// delta, k2q, then the dq and dk/dv kernels, on `stream`.
int launch_backward(const BwdParams& p, const void* out, Strides3 out_st, int D,
                    cudaStream_t stream);

// A selection over blocks of 64 << shift slots rewritten as the same
// selection over 64-slot sub-blocks (sparse_bwd.cu): sub-block 2^shift * c + i
// holds slots 64 i .. 64 i + 63 of block c.  Every listed block becomes its
// sub-blocks that hold real tokens, in order (same keys, same
// multiplicities); query sub-blocks without real rows list nothing.
struct ExpandParams {
  const int32_t* q2k_idx;     // [groups, nq, idx_stride]
  const int32_t* q2k_num;     // [groups, nq]
  const int32_t* q_bs;        // [nq] or null (full blocks)
  const int32_t* kv_bs;       // [nkv] or null
  int32_t* idx64;             // [groups, nq << shift, idx_stride << shift]
  int32_t* num64;             // [groups, nq << shift]
  int32_t* q_bs64;            // [nq << shift]
  int32_t* kv_bs64;           // [nkv << shift]
  long long groups;
  int nq, nkv, idx_stride, shift;
  int* status;
};
int launch_expand_selection(const ExpandParams& e, cudaStream_t stream);

// varlen / metadata helpers (vsa_varlen.cu)
// Logit bound for the entries that take indices (same meaning as
// CoarseParams::qk_bound): block row norms of q and k, then per (group,
// query block) bound_scale * its query norm * the largest key norm among the
// KV blocks it lists in q2k_idx.
struct BoundParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  Strides3 q_st, k_st;
  long long q_seq, kv_seq;    // sequence slots of q and k per (b, h)
  const int32_t* q_tok;       // [nqb] first slot of each query block, or null (64 a)
  const int32_t* kv_tok;      // [nkvb] or null (64 c)
  const int32_t* kv_len;      // [nkvb] real rows, or null (64)
  const int32_t* q_kv_base;   // [nqb] first KV block of the query block's sequence, or null (0)
  const int32_t* q_kv_count;  // [nqb] or null (nkvb)
  const int32_t* q2k_idx;     // [groups, nqb, idx_stride] (indices local to the sequence)
  const int32_t* q2k_num;     // [groups, nqb]
  int idx_stride;
  int B, H, nqb, nkvb;
  int block;                  // slots per block (0: 64)
  float bound_scale;
  float* qn;                  // [groups, nqb]
  float* kn;                  // [groups, nkvb]
  float* qk_bound;            // [groups, nqb]
};
int launch_index_bound(const BoundParams& p, int D, cudaStream_t stream);
// Scratch bytes launch_index_bound needs for its norms and bound.
size_t index_bound_bytes(int groups, int nqb, int nkvb);
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

// Arguments of the whole forward (vsa_forward, vsa_forward_strided and
// vsa_forward_noalloc share the checks and the launch sequence; only the
// layout and the source of the scratch differ).
struct ForwardArgs {
  const void* q;
  const void* k;
  const void* v;
  const void* gate;
  Strides3 q_st, k_st, v_st, out_st, gate_st;
  const int32_t* q_block_sizes;
  const int32_t* kv_block_sizes;
  int B, H, Sq_pad, Skv_pad, D, topk;
  int block;  // slots per block: 64 or 128
  float scale;
  void* out;
  int32_t* q2k_idx;
  int32_t* q2k_num;
  int idx_stride;
  float* out_c;
};
// Strides of contiguous [B, H, S, D] tensors, and of the gate's [B, S, H, D]
// memory seen as a [B, H, S, D] view.
Strides3 bhsd_strides(int H, long long S, int D);
Strides3 gate_strides(int H, long long S, int D);
// Bool block map [rows, nkv] (1 byte per entry, nonzero = selected) to
// ascending q2k_idx rows of width nkv (-1 after the selected blocks) and
// q2k_num.
int launch_mask_to_indices(const uint8_t* block_map, long long rows, int nkv, int32_t* q2k_idx,
                           int32_t* q2k_num, cudaStream_t stream);
// Host checks of vsa_forward's arguments (everything but the workspace).
int check_forward_args(const ForwardArgs& a);
// Pool, coarse + top-k and the sparse kernel with the fused combine, on
// `stream`, with scratch of vsa_forward_workspace_size bytes at `scratch`.
// `profile`: record the profiling events when the hook is set.
int launch_forward(const ForwardArgs& a, void* scratch, bool profile, cudaStream_t stream);

}  // namespace vsa
