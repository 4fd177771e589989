/*
 * vsa.h -- C ABI of the B200 (sm_100a) Video Sparse Attention forward library
 * (libvsa.so).
 *
 * The library computes the VSA forward pass described by the FastVideo pages:
 *   a1 mean-pool q, k, v over 64-slot blocks;
 *   a2 coarse attention among the pooled blocks (out_c, block resolution);
 *   a3 per query block, the top-k KV blocks by coarse logit (q2k_idx, q2k_num);
 *   a4 softmax attention restricted to the selected 64x64 tiles (out_s);
 *   a5 the combine out = out_c * gate + out_s, out_c broadcast inside a block;
 *   a6 a varlen entry over block-aligned packed sequences with rebased indices;
 *   a7 host metadata for 3-D video tiles plus the device token gather/scatter.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Element type "bf16" is IEEE bfloat16 (2 bytes); all activations are bf16.
 * - Layout "BHSD": [batch][head][sequence slot][head dim], contiguous, with the
 *   sequence padded to 64 slots per block: block j occupies slots 64j..64j+63,
 *   its real tokens first.  Padded slots must hold finite values (zeros are
 *   what the packing helpers write); they are never attended to.
 * - Block sizes ("variable_block_sizes") are int32, one per block, each in
 *   [1, 64]; NULL means every block is full (64).  Shared by all batches and
 *   heads.  Sizes outside [1, 64] found on the device set VSA_ERR_BLOCK_SIZE
 *   in the device status word (see vsa_get_device_status).
 * - Head dim D is 64 or 128.
 * - `scale` <= 0 selects 1/sqrt(D).
 * - Pointers documented "device" must point to memory of the current CUDA
 *   device; "host" pointers to ordinary host memory.  The caller owns every
 *   buffer; the library allocates and frees no memory.  Scratch comes from
 *   the caller's `workspace` (size from the matching *_workspace_size call,
 *   256-byte aligned).  (vsa_forward_host creates two copy streams per
 *   device on first use, kept for the process, and a few events per call.)
 * - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls are
 *   asynchronous on that stream and never synchronise it, except
 *   vsa_get_device_status.  The varlen entries (their block tables) and
 *   vsa_forward_host (the block sizes) copy a small host table through a
 *   page-locked staging ring the library keeps per device (8 slots, grown on
 *   first use): the host waits only when the slot it reuses, eight such
 *   calls back, still has its copy in flight.
 * - Every call returns a vsa status code.  Argument problems detectable on
 *   the host are returned before anything is launched.  Problems found inside
 *   kernels (an out-of-range index, a bad block size, a barrier wait that ran
 *   out) are recorded in a per-device status word read by
 *   vsa_get_device_status.  No C++ exception crosses this interface.
 *
 * Page references are to the FastVideo pages: "[kernel] Add varlen support
 * for block-sparse attention" (PR #1319), "[perf] avoid full-sequence
 * materialization in VSA coarse/sparse combine" (PR #1813), "[chore] release
 * fastvideo-kernel 0.3.0" (PR #1478), "[kernel] Extract VSA utility functions
 * into fastvideo_kernel" (PR #1408) and the fastvideo-kernel README.
 */
#ifndef VSA_H_
#define VSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------- */
#define VSA_OK 0
#define VSA_ERR_INVALID_ARG 1    /* null pointer, negative size, bad scale  */
#define VSA_ERR_SHAPE 2          /* inconsistent sizes (e.g. S not 64*n)    */
#define VSA_ERR_UNSUPPORTED 3    /* valid but not built (e.g. D = 96)       */
#define VSA_ERR_CUDA 4           /* a CUDA runtime/driver call failed        */
#define VSA_ERR_DEVICE_TIMEOUT 5 /* a kernel's bounded barrier wait ran out  */
#define VSA_ERR_INDEX_RANGE 6    /* q2k_idx entry outside [0, n_kv_blocks)   */
#define VSA_ERR_WORKSPACE 7      /* workspace missing, small or misaligned   */
#define VSA_ERR_BLOCK_SIZE 8     /* a block size outside [1, 64]             */

/* Largest supported number of KV blocks per sequence and of index entries
 * per query block (the coarse stage keeps a full score row on chip). */
#define VSA_MAX_BLOCKS 2048

/* ---- strided views ------------------------------------------------------ */
/*
 * Element strides (not bytes) of a tensor seen as [batch][head][sequence
 * slot][head dim] with the head dim contiguous.  Every stride of an axis
 * longer than one must be a positive multiple of 8 elements (16 bytes;
 * VSA_ERR_UNSUPPORTED otherwise); a stride of an axis of length one is never
 * used.  Views must not overlap the output.
 */
typedef struct vsa_strides {
  int64_t batch, head, seq;
} vsa_strides;

/* Strides of every tensor of one call.  `gate` describes the gate as a
 * [B, H, Sq, D] view of its memory: for the pages' [B, S, H, D] gate
 * ("compress_attn_weight", passed to the BHSD kernel as a transposed view in
 * PR #1813's follow-up) that is {S*H*D, D, H*D}. */
typedef struct vsa_layout {
  vsa_strides q, k, v, out, gate;
} vsa_layout;

#define VSA_LAYOUT_BHSD 0 /* q, k, v, out contiguous [B, H, S, D] */
#define VSA_LAYOUT_BSHD 1 /* q, k, v, out contiguous [B, S, H, D] */

/* Fill `layout` for contiguous tensors of the given kind; the gate is
 * contiguous [B, Sq_pad, H, D] memory in both kinds.  Host only. */
int vsa_make_layout(int kind, int B, int H, int Sq_pad, int Skv_pad, int D, vsa_layout* layout);

/* Human-readable name of a status code (static string). */
const char* vsa_status_string(int status);

/* Library ABI version: (major << 16) | minor. */
int vsa_abi_version(void);

/*
 * Read and clear the device status word of the current device.
 * Synchronises `stream` first, so it reports every kernel issued before it.
 * Returns VSA_OK or the first error code a kernel recorded since the last
 * read; returns VSA_ERR_CUDA if the synchronisation itself failed.
 */
int vsa_get_device_status(void* stream);

/* ======================================================================== *
 * a1-a5: full VSA forward
 * ======================================================================== */

/*
 * Workspace bytes vsa_forward needs for these sizes, in this order, each
 * region starting on a 256-byte boundary: pooled q [B, H, n_q_blocks, D],
 * pooled k and pooled v [B, H, n_kv_blocks, D], the coarse output when
 * `out_c` is not supplied [B, H, n_q_blocks, D] (all fp32), then fp32 block
 * row norms and a per-query-block bound on the logits, with which the sparse
 * kernel skips its running-max check where the bound proves it unneeded.
 */
size_t vsa_forward_workspace_size(int B, int H, int n_q_blocks, int n_kv_blocks, int D);

/*
 * vsa_forward -- pool, coarse attention, top-k, block-sparse attention and
 * the gated combine, in three kernel launches on `stream`.
 *
 * Defined by: README "Usage" (`video_sparse_attn(q, k, v, block_sizes,
 * block_sizes, topk=5)`); PR #1813 "Problem"/"Change" for the combine
 * out = out_c * gate + out_s with out_c kept at block resolution
 * [B, H, n_blocks, 1, D] and the gate ("compress_attn_weight") laid out
 * [B, S, H, D]; release 0.3.0 "Block-sparse / VSA attention improvements"
 * for q2k_idx / q2k_num.  Readings the pages leave open: coarse softmax
 * scale equals the fine one; top-k ranks scaled coarse logits, ties to the
 * lower KV index, each q2k_idx row ascending with -1 after q2k_num entries;
 * padded query rows of `out` are written as 0.
 *
 * q        device bf16 [B, H, Sq_pad, D]   (Sq_pad = 64 * n_q_blocks)
 * k, v     device bf16 [B, H, Skv_pad, D]  (Skv_pad = 64 * n_kv_blocks)
 * gate     device bf16 [B, Sq_pad, H, D], or NULL for the ungated combine
 *          out = out_c + out_s
 * q_block_sizes   device int32 [Sq_pad/64] or NULL (all 64)
 * kv_block_sizes  device int32 [Skv_pad/64] or NULL (all 64)
 * topk     KV blocks kept per query block, >= 1; clamped to n_kv_blocks
 * out      device bf16 [B, H, Sq_pad, D]
 * q2k_idx  device int32 [B, H, n_q_blocks, idx_stride], written
 * q2k_num  device int32 [B, H, n_q_blocks], written (= min(topk, n_kv))
 * idx_stride  row pitch of q2k_idx, >= min(topk, n_kv_blocks)
 * out_c    device fp32 [B, H, n_q_blocks, D] to receive the coarse output,
 *          or NULL (kept in the workspace)
 * workspace   device, >= vsa_forward_workspace_size(...) bytes, 256-aligned
 *
 * Limits: n_q_blocks, n_kv_blocks in [1, VSA_MAX_BLOCKS]; D in {64, 128}.
 */
int vsa_forward(const void* q, const void* k, const void* v, const void* gate,
                const int32_t* q_block_sizes, const int32_t* kv_block_sizes, int B, int H,
                int Sq_pad, int Skv_pad, int D, int topk, float scale, void* out,
                int32_t* q2k_idx, int32_t* q2k_num, int idx_stride, float* out_c,
                void* workspace, size_t workspace_bytes, void* stream);

/*
 * vsa_forward_strided -- vsa_forward on strided views and either block size:
 * q, k, v, out and gate are read and written through the strides in `layout`
 * (host pointer), so BSHD tensors, slices of a fused QKV tensor and a
 * transposed gate view need no copy.  Same results as vsa_forward on the
 * same values at block_size 64.
 *
 * block_size  slots per block, 64, 128 or 256.  With 128 ("VSA-128":
 *          128-token video tiles), Sq_pad and Skv_pad are multiples of 128,
 *          block sizes lie in [1, 128], pooling and the coarse stage work on
 *          128-slot blocks and the sparse stage attends over 128 x 128
 *          tiles (a kernel shaped for the tensor core's native 128 rows).
 *          With 256 ("VSA-256"), the same on 256-slot blocks (sizes in
 *          [1, 256]); the sparse stage runs the 128-row kernel on each half
 *          of a query block, reading every selected KV block as two 128-key
 *          sub-tiles.
 *
 * Defined by: release 0.3.0, "Block-sparse / VSA attention improvements"
 * (the BSHD-native `video_sparse_attn_bshd` entry and the 128/256-token tile
 * fastpath) and the README's kernel inventory (Blackwell forward kernels for
 * 64- and 128-token blocks); PR #1813's follow-up (the gate passed as a
 * transposed view of its [B, S, H, D] memory).  All other arguments as in
 * vsa_forward with n_q_blocks = Sq_pad / block_size; the workspace size is
 * vsa_forward_workspace_size(B, H, n_q_blocks, n_kv_blocks, D).
 */
int vsa_forward_strided(const void* q, const void* k, const void* v, const void* gate,
                        const vsa_layout* layout, const int32_t* q_block_sizes,
                        const int32_t* kv_block_sizes, int B, int H, int Sq_pad, int Skv_pad,
                        int D, int block_size, int topk, float scale, void* out,
                        int32_t* q2k_idx, int32_t* q2k_num, int idx_stride, float* out_c,
                        void* workspace, size_t workspace_bytes, void* stream);

/*
 * vsa_forward_bshd -- vsa_forward with q, k, v and out contiguous
 * [B, S_pad, H, D] (the layout of release 0.3.0's `video_sparse_attn_bshd`)
 * and the gate [B, Sq_pad, H, D]; arguments otherwise as in vsa_forward.
 */
int vsa_forward_bshd(const void* q, const void* k, const void* v, const void* gate,
                     const int32_t* q_block_sizes, const int32_t* kv_block_sizes, int B, int H,
                     int Sq_pad, int Skv_pad, int D, int topk, float scale, void* out,
                     int32_t* q2k_idx, int32_t* q2k_num, int idx_stride, float* out_c,
                     void* workspace, size_t workspace_bytes, void* stream);

/*
 * vsa_forward_noalloc -- vsa_forward for callers that cannot allocate device
 * memory while they run (a serving loop under a fixed memory budget, where a
 * cudaMalloc can synchronise the device and stall every stream; a plugin
 * whose host application owns all device memory).  The pages have no
 * counterpart to this entry point; it exists for such callers only.
 *
 * Same arguments, results and launches as vsa_forward, minus the workspace:
 * the scratch (vsa_forward's workspace regions, in the same order) lives in
 * one fixed array of VSA_NOALLOC_SCRATCH_BYTES that the
 * library's device image defines.  Every GPU that uses the library holds that
 * array until the process exits.  The call allocates and frees nothing.
 *
 * - Sizes whose scratch exceeds the array, i.e. when
 *   vsa_forward_workspace_size(B, H, n_q_blocks, n_kv_blocks, D) is above
 *   VSA_NOALLOC_SCRATCH_BYTES, return VSA_ERR_WORKSPACE before anything is
 *   launched.  (The H3-like shape B=1, H=56, D=128, 242 + 242 blocks needs
 *   27.9 MB and fits.)
 * - The first call on each device looks the array's device address up and
 *   may load the library's device image there; make that first call before
 *   any stream capture.
 * - All calls on a device share the one array.  Every region of it is
 *   written in full before it is read within a call, so nothing has to be
 *   cleared between calls, but two calls whose kernels overlap on the GPU
 *   (different streams, or different host threads) race on the array and
 *   give wrong results: serialise them, e.g. on one stream.
 */
#define VSA_NOALLOC_SCRATCH_BYTES (32u << 20) /* 32 MiB */
int vsa_forward_noalloc(const void* q, const void* k, const void* v, const void* gate,
                        const int32_t* q_block_sizes, const int32_t* kv_block_sizes, int B, int H,
                        int Sq_pad, int Skv_pad, int D, int topk, float scale, void* out,
                        int32_t* q2k_idx, int32_t* q2k_num, int idx_stride, float* out_c,
                        void* stream);

/*
 * vsa_forward_host -- vsa_forward on tensors in HOST memory.  The library
 * copies the inputs into `workspace` and the results back, in chunks of
 * heads, so that the copies in, the kernels and the copies out of
 * consecutive chunks overlap.  Each chunk is one vsa_forward call (batch of
 * one, the chunk's heads) on the caller's stream, so results equal a single
 * vsa_forward on the same data bit for bit.  The pages define the forward
 * only (see vsa_forward); this entry point is the host-data path around it.
 *
 * q, k, v, gate, out: host, same shapes and types as in vsa_forward.  The
 *          copies overlap the kernels only when these are page-locked
 *          (cudaHostAlloc / cudaHostRegister); pageable memory works but
 *          serialises the copies.  All must stay valid and unchanged until
 *          `stream` has completed the call.
 * q_block_sizes, kv_block_sizes  host int32 or NULL, as in vsa_forward
 * q2k_idx, q2k_num, out_c  host outputs as in vsa_forward, or NULL to skip
 *          copying them back
 * heads_per_chunk  heads per chunk, 0 = about eight chunks in all
 * workspace  device, >= vsa_forward_host_workspace_size(...) bytes,
 *          256-aligned; two chunks' inputs, outputs and forward scratch
 * stream   the caller's stream: the kernels run on it and it waits for the
 *          last copy out, so synchronising it completes the call.  The
 *          copies run on two streams the library keeps per device.
 *
 * Errors are returned before anything is enqueued, except VSA_ERR_CUDA from
 * a failed enqueue, after which part of the work may be queued.
 */
size_t vsa_forward_host_workspace_size(int B, int H, int n_q_blocks, int n_kv_blocks, int D,
                                       int idx_stride, int gated, int heads_per_chunk);
int vsa_forward_host(const void* q, const void* k, const void* v, const void* gate,
                     const int32_t* q_block_sizes, const int32_t* kv_block_sizes, int B, int H,
                     int Sq_pad, int Skv_pad, int D, int topk, float scale, void* out,
                     int32_t* q2k_idx, int32_t* q2k_num, int idx_stride, float* out_c,
                     int heads_per_chunk, void* workspace, size_t workspace_bytes, void* stream);

/* ======================================================================== *
 * a4: block-sparse attention from indices
 * ======================================================================== */

/*
 * block_sparse_attn_from_indices -- out_s = softmax attention of every real
 * query row of block a over the real keys of the KV blocks listed in
 * q2k_idx[b, h, a, 0 : q2k_num[b, h, a]] (a block listed twice counts
 * twice; q2k_num = 0 gives 0).  Padded query rows are written as 0.
 *
 * Defined by: release 0.3.0, "Block-sparse / VSA attention improvements":
 * `block_sparse_attn_from_indices(q, k, v, q2k_idx, q2k_num,
 * variable_block_sizes)`, the index-native block-sparse API.
 *
 * q, k, v, q_block_sizes, kv_block_sizes, Sq_pad, Skv_pad, D, scale: as in
 *          vsa_forward
 * q2k_idx  device int32 [B, H, n_q_blocks, idx_stride]; entries past
 *          q2k_num are ignored.  An entry outside [0, n_kv_blocks) is
 *          skipped and sets VSA_ERR_INDEX_RANGE in the device status word.
 * q2k_num  device int32 [B, H, n_q_blocks], each in [0, idx_stride]
 * idx_stride  1 .. VSA_MAX_BLOCKS
 * out      device bf16 [B, H, Sq_pad, D]
 * lse      device fp32 [B, H, Sq_pad] or NULL: the natural-log
 *          log-sum-exp of each real query row's scaled logits over its
 *          selected keys (-inf where nothing is selected, 0 on padded rows),
 *          the softmax normaliser block_sparse_attn_backward(_ex) takes.
 *          Any block size (ABI 2.1; 2.0 took it at block size 64 only).
 * layout   host, strides of q, k, v and out (gate unused), or NULL for
 *          contiguous BHSD
 * workspace  device, >= block_sparse_attn_from_indices_workspace_size(...)
 *          bytes, 256-aligned, or NULL.  With it, one extra pass takes block
 *          row norms of q and k and bounds every query block's logits by
 *          its query norm times the largest key norm among the blocks it
 *          lists; where the bound shows no logit can exceed the first tile
 *          pair's maxima by 2^32, the sparse kernel skips its running-max
 *          check, and where the bound is at most 60 (log2 units) it serves
 *          as the reference max from the first step on (fewer instructions;
 *          the results equal those without the workspace up to the rounding
 *          of the probabilities).  Without it every step keeps the check.
 * block_size  64, 128 or 256 (see vsa_forward_strided); n_q_blocks =
 *          Sq_pad / block_size
 * (ABI 2.0 added layout, block_size and workspace.)
 */
size_t block_sparse_attn_from_indices_workspace_size(int B, int H, int n_q_blocks,
                                                     int n_kv_blocks);
int block_sparse_attn_from_indices(const void* q, const void* k, const void* v,
                                   const int32_t* q2k_idx, const int32_t* q2k_num,
                                   const int32_t* q_block_sizes, const int32_t* kv_block_sizes,
                                   int B, int H, int Sq_pad, int Skv_pad, int D, int block_size,
                                   int idx_stride, float scale, void* out, float* lse,
                                   const vsa_layout* layout, void* workspace,
                                   size_t workspace_bytes, void* stream);

/*
 * block_sparse_attn -- block-sparse attention from a bool block map:
 * block_map[b, h, a, c] != 0 selects KV block c for query block a.  The map
 * is converted on the device to ascending index rows, written to q2k_idx
 * (row width n_kv_blocks, -1 after the selected blocks) and q2k_num, and
 * those run exactly as in block_sparse_attn_from_indices (so the results are
 * bit-identical to that call on the same indices).
 *
 * Defined by: release 0.3.0, "Block-sparse / VSA attention improvements" and
 * "New / changed public API": the legacy `block_sparse_attn(..., block_map,
 * ...)` bool-mask API kept as a wrapper over the index-native kernel.
 *
 * block_map  device uint8 (torch.bool) [B, H, n_q_blocks, n_kv_blocks]
 * q2k_idx    device int32 [B, H, n_q_blocks, n_kv_blocks], written
 * q2k_num    device int32 [B, H, n_q_blocks], written
 * everything else as in block_sparse_attn_from_indices (the workspace size
 * is block_sparse_attn_from_indices_workspace_size's).
 */
int block_sparse_attn(const void* q, const void* k, const void* v, const uint8_t* block_map,
                      const int32_t* q_block_sizes, const int32_t* kv_block_sizes, int B, int H,
                      int Sq_pad, int Skv_pad, int D, int block_size, float scale, void* out,
                      int32_t* q2k_idx, int32_t* q2k_num, const vsa_layout* layout,
                      void* workspace, size_t workspace_bytes, void* stream);

/* ======================================================================== *
 * a6: varlen block-sparse attention
 * ======================================================================== */

/* Workspace bytes for block_sparse_attn_varlen: the device block tables,
 * then fp32 block row norms of q and k and a per-(head, query block) bound
 * on the logits, with which the sparse kernel skips its running-max check
 * where the bound proves it unneeded (H heads).  (ABI 1.1 added H.) */
size_t block_sparse_attn_varlen_workspace_size(int n_seqs, int total_q_blocks,
                                               int total_kv_blocks, int H);

/*
 * block_sparse_attn_varlen -- block-sparse attention over several sequences
 * of different lengths in one launch.
 *
 * Defined by: PR #1319 "How it works": sequences are packed block-aligned
 * (each block takes 64 slots), each sequence's q2k_idx is rebased to global
 * block offsets, one block-sparse call covers the whole batch, and the output
 * is unpacked per sequence; Q and KV lengths may differ (release 0.3.0,
 * "Varlen block-sparse attention").  Here the packing is virtual: a device
 * block table gives each packed block's first token, so the kernel reads the
 * token-packed inputs in place and writes only real rows of `out`.
 *
 * q        device bf16 [H, total_q, D], sequences back to back
 * k, v     device bf16 [H, total_kv, D]
 * cu_seqlens_q, cu_seqlens_kv  host int32 [n_seqs + 1], non-decreasing,
 *          starting at 0; total_q = cu_seqlens_q[n_seqs]
 * q_block_sizes   host int32, the blocks of every sequence concatenated
 *          (each in [1, 64], per sequence summing to its length), or NULL:
 *          64-token blocks with a partial last block
 * cu_q_blocks     host int32 [n_seqs + 1]: first block of each sequence in
 *          q_block_sizes; required iff q_block_sizes is given
 * kv_block_sizes, cu_kv_blocks  the same for K/V
 * q2k_idx  device int32 [H, total_q_blocks, idx_stride]: rows of sequence i
 *          hold indices local to sequence i's KV blocks
 * q2k_num  device int32 [H, total_q_blocks]
 * out      device bf16 [H, total_q, D]; only real token rows are written
 * lse      device fp32 [H, total_q] or NULL: per real token row the
 *          natural-log log-sum-exp of its scaled logits (see
 *          block_sparse_attn_from_indices)
 * pack_index_q   device int64 [64 * total_q_blocks] or NULL: for each packed
 *          slot the token row of q it holds, -1 for padding
 * pack_index_kv  device int64 [64 * total_kv_blocks] or NULL: same for k/v
 * q2k_idx_rebased  device int32 [H, total_q_blocks, idx_stride] or NULL:
 *          q2k_idx plus each sequence's first packed KV block, -1 tails
 * workspace  device, >= block_sparse_attn_varlen_workspace_size(...) bytes
 *
 * Host checks return VSA_ERR_SHAPE for an empty batch, a sequence with zero
 * tokens, or block sizes whose count or sum disagrees with the lengths (the
 * PR #1319 review notes).
 */
int block_sparse_attn_varlen(const void* q, const void* k, const void* v,
                             const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_kv,
                             const int32_t* q_block_sizes, const int32_t* cu_q_blocks,
                             const int32_t* kv_block_sizes, const int32_t* cu_kv_blocks,
                             int n_seqs, int H, int D, const int32_t* q2k_idx,
                             const int32_t* q2k_num, int idx_stride, float scale, void* out,
                             float* lse, int64_t* pack_index_q, int64_t* pack_index_kv,
                             int32_t* q2k_idx_rebased, void* workspace, size_t workspace_bytes,
                             void* stream);

/* ======================================================================== *
 * backward of the block-sparse attention (64-slot blocks; any block size
 * through block_sparse_attn_backward_ex)
 * ======================================================================== */

/*
 * Workspace bytes block_sparse_attn_backward needs: fp32 delta (sum over
 * the head dim of dout * out) per query row [B, H, Sq_pad], then the k2q
 * index (for every KV block the query blocks that selected it, with their
 * multiplicities) [B, H, n_kv_blocks, Sq_pad / 64] and its counts.
 */
size_t block_sparse_attn_backward_workspace_size(int B, int H, int Sq_pad, int n_kv_blocks);

/*
 * block_sparse_attn_backward -- dq, dk, dv of block_sparse_attn_from_indices
 * (block size 64) for the output gradient dout.
 *
 * Defined by: PR #1319 "Summary" / "Backward correctness" (dQ/dK/dV of the
 * block-sparse attention; the backward goes through a k2q index, KV block
 * -> query blocks) and release 0.3.0 ("Supports forward and backward").
 * With P = softmax(scale * q k^T) over each query block's selected keys (a
 * block listed twice counts twice): dv = P^T dout, dS = P * (dout v^T -
 * rowsum(dout * out)), dq = scale * dS k, dk = scale * dS^T q.  Padded rows
 * of dq, dk, dv are written as 0; keys no query block selected get 0.
 *
 * q, k, v, q2k_idx, q2k_num, block sizes, sizes, scale: as in the forward
 *          call (contiguous BHSD)
 * out      device bf16 [B, H, Sq_pad, D]: that call's output
 * dout     device bf16 [B, H, Sq_pad, D]
 * lse      device fp32 [B, H, Sq_pad]: that call's log-sum-exp output
 * dq       device bf16 [B, H, Sq_pad, D], written
 * dk, dv   device bf16 [B, H, Skv_pad, D], written
 * workspace  device, >= block_sparse_attn_backward_workspace_size(...),
 *          256-aligned
 * Four launches on `stream`: delta, k2q, the dq pass and the dk/dv pass.
 */
int block_sparse_attn_backward(const void* q, const void* k, const void* v, const void* out,
                               const void* dout, const float* lse, const int32_t* q2k_idx,
                               const int32_t* q2k_num, const int32_t* q_block_sizes,
                               const int32_t* kv_block_sizes, int B, int H, int Sq_pad,
                               int Skv_pad, int D, int idx_stride, float scale, void* dq,
                               void* dk, void* dv, void* workspace, size_t workspace_bytes,
                               void* stream);

/*
 * Workspace bytes block_sparse_attn_backward_ex needs: those of
 * block_sparse_attn_backward_workspace_size(B, H, Sq_pad, Skv_pad / 64),
 * then for block_size 128 / 256 the selection rewritten over 64-slot
 * sub-blocks: int32 index rows [B, H, Sq_pad / 64, idx_stride * r], counts
 * [B, H, Sq_pad / 64], query and key sub-block sizes (r = block_size / 64).
 * 0 for invalid arguments.  (ABI 2.1.)
 */
size_t block_sparse_attn_backward_ex_workspace_size(int B, int H, int Sq_pad, int Skv_pad,
                                                    int block_size, int idx_stride);

/*
 * block_sparse_attn_backward_ex -- block_sparse_attn_backward for a forward
 * call of any block size (64, 128 or 256; ABI 2.1).
 *
 * Defined by: PR #1319 "Summary" / "Backward correctness" as for
 * block_sparse_attn_backward, at the tile sizes of release 0.3.0's 128/256
 * tile fastpath ("Block-sparse / VSA attention improvements").  The gradients of attention over a list of blocks depend only on
 * which key rows each query row sees, so a selection over blocks of
 * 64 r slots equals the selection over their 64-slot sub-blocks: a first
 * launch rewrites it on the device (every listed block c becomes its
 * sub-blocks r c + i that hold real keys, i = 0 .. r - 1, in order, with the
 * same multiplicity; each query sub-block with real rows lists them all,
 * the others nothing), then the four launches of block_sparse_attn_backward
 * run on it.  The results equal those of the 64-slot call on that rewritten
 * selection bit for bit.
 *
 * Arguments as in block_sparse_attn_backward, plus
 * block_size  64, 128 or 256: that of the forward call; q2k_idx, q2k_num,
 *          q_block_sizes, kv_block_sizes are in its blocks (Sq_pad /
 *          block_size query blocks, Skv_pad / block_size KV blocks)
 * Limits: idx_stride * block_size / 64, Sq_pad / 64 and Skv_pad / 64 at most
 * VSA_MAX_BLOCKS (else VSA_ERR_UNSUPPORTED).
 * workspace  device, >= block_sparse_attn_backward_ex_workspace_size(...),
 *          256-aligned
 * Five launches on `stream` for block size 128 / 256, four for 64.
 */
int block_sparse_attn_backward_ex(const void* q, const void* k, const void* v, const void* out,
                                  const void* dout, const float* lse, const int32_t* q2k_idx,
                                  const int32_t* q2k_num, const int32_t* q_block_sizes,
                                  const int32_t* kv_block_sizes, int B, int H, int Sq_pad,
                                  int Skv_pad, int D, int block_size, int idx_stride, float scale,
                                  void* dq, void* dk, void* dv, void* workspace,
                                  size_t workspace_bytes, void* stream);

/* Workspace bytes block_sparse_attn_varlen_backward needs: the block tables,
 * delta per packed query row [H, total_q] and the k2q index over the packed
 * blocks. */
size_t block_sparse_attn_varlen_backward_workspace_size(int n_seqs, int total_q_blocks,
                                                        int total_kv_blocks, int H, int total_q);

/*
 * block_sparse_attn_varlen_backward -- dq, dk, dv of block_sparse_attn_varlen
 * (PR #1319: the varlen backward through a k2q index; "dQ/dK/dV match
 * per-sequence reference exactly").  Arguments as in the forward varlen call
 * plus out and lse from it (lse [H, total_q]), dout [H, total_q, D] and the
 * outputs dq [H, total_q, D], dk, dv [H, total_kv, D] (real token rows
 * written).
 */
int block_sparse_attn_varlen_backward(
    const void* q, const void* k, const void* v, const void* out, const void* dout, const float* lse,
    const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_kv, const int32_t* q_block_sizes,
    const int32_t* cu_q_blocks, const int32_t* kv_block_sizes, const int32_t* cu_kv_blocks,
    int n_seqs, int H, int D, const int32_t* q2k_idx, const int32_t* q2k_num, int idx_stride,
    float scale, void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes,
    void* stream);

/* ======================================================================== *
 * a7: video tile metadata (host) and token gather / scatter (device)
 * ======================================================================== */

/*
 * build_vsa_metadata -- tile partition of a T x Hh x W latent (tokens
 * numbered row-major over (t, h, w)) into tT x tH x tW tiles.
 *
 * Defined by: PR #1408 "Summary"/"Design decisions": one call builds
 * tile_partition_indices, reverse_tile_partition_indices, the variable block
 * sizes (tokens per tile, at most the tile volume, tile size a parameter)
 * and the non-pad index (get_non_pad_index(variable_block_sizes,
 * max_block_size)).  The pages name these but not the order; this library
 * visits tiles in row-major (t, h, w) tile order, tokens inside a tile in
 * row-major (t, h, w) order, and clips edge tiles.
 *
 * All pointers are host memory.  Outputs may be NULL to skip them; call
 * first with all outputs NULL except n_tiles to size the arrays.
 * tile_partition_indices          int64 [T*Hh*W]: token at tiled position j
 * reverse_tile_partition_indices  int64 [T*Hh*W]: tiled position of token i
 * variable_block_sizes            int32 [n_tiles]
 * non_pad_index                   int64 [T*Hh*W]: padded slot of tiled
 *                                 position j (tile volume slots per tile)
 * slot_token                      int64 [n_tiles * tT*tH*tW]: token held by
 *                                 each padded slot, -1 for padding
 * n_tiles                         int32 [1]
 * Returns VSA_ERR_INVALID_ARG for non-positive sizes or a tile volume above
 * 256 (64 for the 64-slot path, 128 or 256 for VSA-128 / VSA-256 tiles such
 * as 4 x 4 x 8 or 4 x 8 x 8).
 */
int build_vsa_metadata(int T, int Hh, int W, int tT, int tH, int tW,
                       int64_t* tile_partition_indices, int64_t* reverse_tile_partition_indices,
                       int32_t* variable_block_sizes, int64_t* non_pad_index,
                       int64_t* slot_token, int32_t* n_tiles);

/*
 * vsa_gather_tokens -- dst[g, s, :] = src[g, slot_token[s], :], or 0 where
 * slot_token[s] < 0: places tokens into the tiled, padded block layout.
 * src device bf16 [groups, n_tokens, D]; dst device bf16 [groups, n_slots, D];
 * slot_token device int64 [n_slots] with entries < n_tokens.
 * (PR #1408: the tile permutation plus non-pad placement the metadata
 * describes.)
 */
int vsa_gather_tokens(const void* src, void* dst, const int64_t* slot_token, int64_t n_tokens,
                      int64_t n_slots, int64_t groups, int D, void* stream);

/*
 * vsa_scatter_tokens -- dst[g, slot_token[s], :] = src[g, s, :] for every
 * slot with slot_token[s] >= 0: the inverse of vsa_gather_tokens on the real
 * tokens.  Same argument meanings; dst is [groups, n_tokens, D].
 */
int vsa_scatter_tokens(const void* src, void* dst, const int64_t* slot_token, int64_t n_tokens,
                       int64_t n_slots, int64_t groups, int D, void* stream);

/* ======================================================================== *
 * head-sharded multi-GPU path: resharding around the all-to-all exchanges
 * ======================================================================== */

/*
 * vsa_permute_rows -- copy rows of D bf16 elements: destination row
 * ((a0 * E1 + a1) * E2 + a2) * E3 + a3 (a_i < E_i, extents[i] = E_i) takes
 * source row a0 * S0 + a1 * S1 + a2 * S2 + a3 * S3 (src_strides[i] = S_i,
 * in rows).  Every reshard of the sequence-parallel ("Ulysses") wrapper is
 * one such call: a rank's sequence shard [B, S_local, H, D] packed into
 * per-destination head groups [N, B, S_local, H/N, D] before the first
 * all-to-all, the received shards gathered into [B, S, H/N, D], and the
 * reverse two after the forward.
 *
 * Defined by: README "Compiled CUDA extensions" (the fused NVLink Ulysses
 * all-to-all that reshards between sequence and head parallelism) and the
 * 4-GPU sequence-parallel recipe it serves; the exchange itself is NCCL's.
 *
 * src, dst   device bf16; src must hold every row the strides reach, dst
 *            E0 * E1 * E2 * E3 rows; both 16-byte aligned, not overlapping
 * extents    host int64 [4]; E0, E1 <= 65535
 * src_strides host int64 [4], >= 0
 * D          a multiple of 8
 */
int vsa_permute_rows(const void* src, void* dst, const int64_t* extents,
                     const int64_t* src_strides, int D, void* stream);

/* ======================================================================== *
 * diagnostics
 * ======================================================================== */

/*
 * vsa_set_profile_events -- timing hook for vsa_forward.  `events` points to
 * four cudaEvent_t handles (host array) or is NULL to switch the hook off.
 * While set, every vsa_forward call records events[0] on its stream before
 * the pooling kernel, events[1] after it, events[2] after the coarse/top-k
 * kernel and events[3] after the block-sparse kernel, so a caller can time
 * each kernel with cudaEventElapsedTime.  The handles are copied; the setting
 * is process-wide and not thread-safe.
 */
int vsa_set_profile_events(void* const* events);

/*
 * vsa_selftest_umma -- run the tensor-core products of the sparse kernels
 * once on operands in global memory, to check shared-memory and TMEM
 * layouts in isolation.  64-slot kernel: mode 0: c[128][64] = a[128][D] *
 * b[64][D]^T (fp32), the transposed-score product; mode 1: c[D][64] =
 * a[128][D]^T * b[128][64], the transposed-output product.  128-slot
 * kernel: mode 2: c[128][128] = a[128][D] * b[128][D]^T; mode 3: c[128][D] =
 * a[128][128] * b[128][D] with a staged in TMEM.  a, b device bf16; c device
 * fp32.  D 64 or 128.
 */
int vsa_selftest_umma(int mode, int D, const void* a, const void* b, float* c, void* stream);

/*
 * vsa_selftest_exp2 -- evaluate the sparse kernel's FMA-pipe exponential
 * (2^x by range reduction and a fitted cubic; the pages fix no such routine,
 * it is an implementation detail of the softmax) on x[0 .. n): y[i] is its
 * value, and *mismatch (device int32, added to) counts elements where the two
 * halves of the packed evaluation disagree.  x, y device fp32 [n].
 */
int vsa_selftest_exp2(const float* x, float* y, int64_t n, int* mismatch, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* VSA_H_ */
