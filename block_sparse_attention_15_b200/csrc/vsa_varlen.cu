// a6 varlen side outputs (pack indices, rebased q2k_idx) and a7 token
// gather / scatter between the token order and the tiled, padded block
// layout.  All three are index/copy work: coalesced 16-byte moves, one thread
// per element or per 16-byte chunk.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "vsa.h"
#include "vsa_device.cuh"
#include "vsa_launch.h"

namespace vsa {

// pack_index[64*blk + t] = first token row of blk + t for t < len(blk), else -1
// ("[kernel] Add varlen support for block-sparse attention", How it works,
// step 1: each block occupies 64 slots).
__global__ void pack_index_kernel(const int32_t* blk_tok, const int32_t* blk_len, int n_blocks,
                                  int64_t* pack_index) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= 64LL * n_blocks) return;
  const int blk = (int)(i / 64), t = (int)(i % 64);
  pack_index[i] = (t < blk_len[blk]) ? (int64_t)blk_tok[blk] + t : (int64_t)-1;
}

// Step 2 of the same section: per-sequence KV block indices shifted to the
// sequence's first packed KV block.  Entries past q2k_num become -1.
__global__ void rebase_kernel(const int32_t* q2k_idx, const int32_t* q2k_num,
                              const int32_t* q_kv_base, const int32_t* q_kv_count, int H, int nq,
                              int idx_stride, int32_t* out, int* status) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long total = (long long)H * nq * idx_stride;
  if (i >= total) return;
  const long long rowid = i / idx_stride;  // h * nq + a
  const int j = (int)(i % idx_stride);
  const int a = (int)(rowid % nq);
  const int num = q2k_num[rowid];
  int32_t v = -1;
  if (j < num) {
    const int c = q2k_idx[i];
    if (c < 0 || c >= q_kv_count[a]) {
      set_status(status, VSA_ERR_INDEX_RANGE);
    } else {
      v = c + q_kv_base[a];
    }
  }
  out[i] = v;
}

template <bool SCATTER>
__global__ void gather_tokens_kernel(const uint4* src, uint4* dst, const int64_t* slot_token,
                                     int64_t n_tokens, int64_t n_slots, int64_t groups,
                                     int chunks) {
  const long long total = groups * n_slots * chunks;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int ch = (int)(i % chunks);
    const long long gs = i / chunks;
    const long long s = gs % n_slots, g = gs / n_slots;
    const int64_t tok = slot_token[s];
    if (!SCATTER) {
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (tok >= 0 && tok < n_tokens) v = __ldcs(src + ((g * n_tokens + tok) * chunks + ch));
      __stcs(dst + i, v);
    } else if (tok >= 0 && tok < n_tokens) {
      __stcs(dst + ((g * n_tokens + tok) * chunks + ch), __ldcs(src + i));
    }
  }
}

int launch_varlen_aux(const int32_t* blk_tok, const int32_t* blk_len, int n_blocks,
                      int64_t* pack_index, cudaStream_t stream) {
  const long long n = 64LL * n_blocks;
  if (n <= 0) return VSA_OK;
  pack_index_kernel<<<(unsigned)((n + 255) / 256), 256, 0, stream>>>(blk_tok, blk_len, n_blocks,
                                                                       pack_index);
  return cudaGetLastError() == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

int launch_rebase(const int32_t* q2k_idx, const int32_t* q2k_num, const int32_t* q_kv_base,
                  const int32_t* q_kv_count, int H, int nq, int idx_stride, int32_t* out,
                  int* status, cudaStream_t stream) {
  const long long n = (long long)H * nq * idx_stride;
  if (n <= 0) return VSA_OK;
  rebase_kernel<<<(unsigned)((n + 255) / 256), 256, 0, stream>>>(
      q2k_idx, q2k_num, q_kv_base, q_kv_count, H, nq, idx_stride, out, status);
  return cudaGetLastError() == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

int launch_gather_tokens(const void* src, void* dst, const int64_t* slot_token, int64_t n_tokens,
                         int64_t n_slots, int64_t groups, int D, bool scatter,
                         cudaStream_t stream) {
  const int chunks = D / 8;
  const long long total = groups * n_slots * chunks;
  if (total <= 0) return VSA_OK;
  int sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) {
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  }
  long long blocks = (total + 255) / 256;
  const long long cap = (long long)sms * 8;  // 8 resident CTAs of 256 threads per SM
  if (blocks > cap) blocks = cap;
  if (scatter) {
    gather_tokens_kernel<true><<<(unsigned)blocks, 256, 0, stream>>>(
        static_cast<const uint4*>(src), static_cast<uint4*>(dst), slot_token, n_tokens, n_slots,
        groups, chunks);
  } else {
    gather_tokens_kernel<false><<<(unsigned)blocks, 256, 0, stream>>>(
        static_cast<const uint4*>(src), static_cast<uint4*>(dst), slot_token, n_tokens, n_slots,
        groups, chunks);
  }
  return cudaGetLastError() == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

}  // namespace vsa
