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

// One CTA per (SPB * kSlotsPerThread slots, kGroupsPerCta groups): thread t
// moves 16-byte chunk t % (D / 8) of kSlotsPerThread slots spaced SPB apart,
// for each of the CTA's groups.  The slot indices are loaded once for all
// the groups, then every data load of the groups is issued, then every
// store: a gather's two dependent loads (index, then token row) pay the
// index latency once per kGroupsPerCta groups, with kSlotsPerThread *
// kGroupsPerCta loads in flight per thread.
constexpr int kSlotsPerThread = 4;
constexpr int kGroupsPerCta = 4;

template <bool SCATTER, int D>
__global__ void __launch_bounds__(256) gather_tokens_kernel(const uint4* src, uint4* dst,
                                                            const int64_t* slot_token,
                                                            int n_tokens, int n_slots, int groups) {
  constexpr int CH = D / 8;             // 16-byte chunks per row
  constexpr int SPB = 256 / CH;         // slots per pass
  const int ch = (int)threadIdx.x % CH;
  const int s0 = blockIdx.x * SPB * kSlotsPerThread + (int)threadIdx.x / CH;
  const int g0 = blockIdx.y * kGroupsPerCta;
  int tok[kSlotsPerThread];
#pragma unroll
  for (int i = 0; i < kSlotsPerThread; ++i) {
    const int s = s0 + i * SPB;
    const int64_t t = s < n_slots ? slot_token[s] : -1;
    tok[i] = (t >= 0 && t < n_tokens) ? (int)t : -1;  // -1: padding (or out of range)
  }
  uint4 v[kGroupsPerCta][kSlotsPerThread];
#pragma unroll
  for (int k = 0; k < kGroupsPerCta; ++k) {
    const long long g = g0 + k;
    const uint4* sg = src + g * (SCATTER ? n_slots : n_tokens) * CH + ch;
#pragma unroll
    for (int i = 0; i < kSlotsPerThread; ++i) {
      const int s = s0 + i * SPB;
      v[k][i] = make_uint4(0u, 0u, 0u, 0u);
      if (g < groups && s < n_slots && tok[i] >= 0)
        v[k][i] = __ldcs(sg + (long long)(SCATTER ? s : tok[i]) * CH);
    }
  }
#pragma unroll
  for (int k = 0; k < kGroupsPerCta; ++k) {
    const long long g = g0 + k;
    if (g >= groups) break;
    uint4* dg = dst + g * (SCATTER ? n_tokens : n_slots) * CH + ch;
#pragma unroll
    for (int i = 0; i < kSlotsPerThread; ++i) {
      const int s = s0 + i * SPB;
      if (s >= n_slots) continue;
      if (!SCATTER) __stcs(dg + (long long)s * CH, v[k][i]);
      else if (tok[i] >= 0) __stcs(dg + (long long)tok[i] * CH, v[k][i]);
    }
  }
}

// Largest row L2 norm of one block per (group, block): query blocks over the
// block's slots from its first token (the rows the sparse kernel's query
// tiles hold, clipped at the end of the sequence), key blocks over their real
// rows.  One CTA of 256 threads per (group, block), 64 rows at a time; the
// squared norms of a row's D/8 16-byte chunks add up across consecutive lanes.
template <int D>
__global__ void __launch_bounds__(256, 8) block_norm_kernel(BoundParams p) {
  constexpr int CPR = D / 8, RPP = 256 / CPR, PASSES = 64 / RPP;
  const int bsz = p.block > 0 ? p.block : 64;
  __shared__ float wmax[8];
  const long long item = blockIdx.x;  // group * (nqb + nkvb) + block
  const int per_group = p.nqb + p.nkvb;
  const long long group = item / per_group;
  const int blk = (int)(item % per_group);
  const int b = (int)(group / p.H), h = (int)(group % p.H);
  const bool is_q = blk < p.nqb;
  const __nv_bfloat16* base;
  long long s0, s_end, st;
  int rows;
  float* dst;
  if (is_q) {
    base = p.q + b * p.q_st.b + h * p.q_st.h;
    st = p.q_st.s;
    s0 = p.q_tok ? p.q_tok[blk] : (long long)bsz * blk;
    s_end = p.q_seq;
    rows = bsz;
    dst = p.qn + group * p.nqb + blk;
  } else {
    const int c = blk - p.nqb;
    base = p.k + b * p.k_st.b + h * p.k_st.h;
    st = p.k_st.s;
    s0 = p.kv_tok ? p.kv_tok[c] : (long long)bsz * c;
    s_end = p.kv_seq;
    rows = p.kv_len ? p.kv_len[c] : bsz;
    rows = rows < 0 ? 0 : (rows > bsz ? bsz : rows);
    dst = p.kn + group * p.nkvb + c;
  }
  const int chunk = threadIdx.x % CPR, r0 = threadIdx.x / CPR;
  float mx = 0.f;
#pragma unroll 1
  for (int c0 = 0; c0 < rows; c0 += 64) {
  uint4 buf[PASSES];  // every load of the chunk issued before any use
#pragma unroll
  for (int ps = 0; ps < PASSES; ++ps) {
    const int r = c0 + r0 + ps * RPP;
    buf[ps] = (r < rows && s0 + r < s_end)
                  ? __ldcs(reinterpret_cast<const uint4*>(base + (s0 + r) * st) + chunk)
                  : make_uint4(0u, 0u, 0u, 0u);
  }
#pragma unroll
  for (int ps = 0; ps < PASSES; ++ps) {
    const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&buf[ps]);
    float sq = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(h2[e]);
      sq = fmaf(f.x, f.x, sq);
      sq = fmaf(f.y, f.y, sq);
    }
#pragma unroll
    for (int o = CPR / 2; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
    mx = fmaxf(mx, sq);
  }
  }
#pragma unroll
  for (int o = CPR; o < 32; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = mx;
  __syncthreads();
  if (threadIdx.x == 0) {
    float m = wmax[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) m = fmaxf(m, wmax[w]);
    *dst = __fsqrt_rn(m);
  }
}

// Per (group, query block): bound_scale * its query norm * the largest key
// norm among the KV blocks its q2k_idx row lists (entries outside the
// sequence's blocks are skipped here; the sparse kernel reports them).  A
// tighter bound than the largest key norm of the whole head, so more items
// take the vote-free step.
__global__ void index_bound_kernel(BoundParams p) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (long long)p.B * p.H * p.nqb) return;
  const long long group = i / p.nqb;
  const int a = (int)(i % p.nqb);
  const int base = p.q_kv_base ? p.q_kv_base[a] : 0;
  const int count = p.q_kv_count ? p.q_kv_count[a] : p.nkvb;
  const float* kn = p.kn + group * p.nkvb + base;
  const int32_t* idx = p.q2k_idx + i * p.idx_stride;
  int num = p.q2k_num[i];
  num = num < 0 ? 0 : (num > p.idx_stride ? p.idx_stride : num);
  float km = 0.f;
  for (int j = 0; j < num; ++j) {
    const int c = idx[j];
    if (c >= 0 && c < count) km = fmaxf(km, kn[c]);
  }
  p.qk_bound[i] = p.bound_scale * p.qn[i] * km;
}

size_t index_bound_bytes(int groups, int nqb, int nkvb) {
  return sizeof(float) * (size_t)groups * (2 * (size_t)nqb + nkvb);
}

int launch_index_bound(const BoundParams& p, int D, cudaStream_t stream) {
  const long long groups = (long long)p.B * p.H;
  const long long grid = groups * (p.nqb + p.nkvb);
  if (grid <= 0) return VSA_OK;
  if (grid > 0x7FFFFFFFLL) return VSA_ERR_UNSUPPORTED;
  if (D == 128) block_norm_kernel<128><<<(unsigned)grid, 256, 0, stream>>>(p);
  else block_norm_kernel<64><<<(unsigned)grid, 256, 0, stream>>>(p);
  if (cudaGetLastError() != cudaSuccess) return VSA_ERR_CUDA;
  const long long n = groups * p.nqb;
  index_bound_kernel<<<(unsigned)((n + 255) / 256), 256, 0, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

// One warp per row of the block map: the selected KV blocks in ascending
// order by ballot compaction, 32 columns at a time ("[chore] release
// fastvideo-kernel 0.3.0", Block-sparse / VSA attention improvements: the
// legacy bool block_map API becomes a wrapper over the index-native kernel).
__global__ void __launch_bounds__(256) mask_to_indices_kernel(const uint8_t* block_map, long long rows,
                                                              int nkv, int32_t* q2k_idx,
                                                              int32_t* q2k_num) {
  const long long row = (long long)blockIdx.x * 8 + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (row >= rows) return;
  const uint8_t* m = block_map + row * nkv;
  int32_t* out = q2k_idx + row * nkv;
  int n = 0;
  for (int c0 = 0; c0 < nkv; c0 += 32) {
    const int c = c0 + lane;
    const bool sel = c < nkv && m[c] != 0;
    const uint32_t ball = __ballot_sync(0xffffffffu, sel);
    if (sel) out[n + __popc(ball & ((1u << lane) - 1u))] = c;
    n += __popc(ball);
  }
  for (int j = n + lane; j < nkv; j += 32) out[j] = -1;
  if (lane == 0) q2k_num[row] = n;
}

int launch_mask_to_indices(const uint8_t* block_map, long long rows, int nkv, int32_t* q2k_idx,
                           int32_t* q2k_num, cudaStream_t stream) {
  if (rows <= 0 || nkv <= 0) return VSA_OK;
  const long long grid = (rows + 7) / 8;
  if (grid > 0x7FFFFFFFLL) return VSA_ERR_UNSUPPORTED;
  mask_to_indices_kernel<<<(unsigned)grid, 256, 0, stream>>>(block_map, rows, nkv, q2k_idx, q2k_num);
  return cudaGetLastError() == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
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

// Any other row width (D a multiple of 8): one CTA per (slot, group), the
// threads striding over the row's chunks.
template <bool SCATTER>
__global__ void __launch_bounds__(256) gather_tokens_any_kernel(const uint4* src, uint4* dst,
                                                                const int64_t* slot_token,
                                                                int n_tokens, int n_slots, int CH) {
  const int s = blockIdx.x;
  const long long g = blockIdx.y;
  const int64_t tok = slot_token[s];
  const bool real = tok >= 0 && tok < n_tokens;
  for (int ch = threadIdx.x; ch < CH; ch += blockDim.x) {
    const long long slot_i = (g * n_slots + s) * CH + ch;
    if (!SCATTER) {
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (real) v = __ldcs(src + ((g * n_tokens + tok) * CH + ch));
      __stcs(dst + slot_i, v);
    } else if (real) {
      __stcs(dst + ((g * n_tokens + tok) * CH + ch), __ldcs(src + slot_i));
    }
  }
}

int launch_gather_tokens(const void* src, void* dst, const int64_t* slot_token, int64_t n_tokens,
                         int64_t n_slots, int64_t groups, int D, bool scatter,
                         cudaStream_t stream) {
  if (groups <= 0 || n_slots <= 0) return VSA_OK;
  if (n_tokens > 0x7FFFFFFFLL || n_slots > 0x7FFFFFFFLL || groups > 65535) return VSA_ERR_UNSUPPORTED;
  const int spb = D <= 2048 ? 256 / (D / 8) * kSlotsPerThread : 1;
  const dim3 grid((unsigned)((n_slots + spb - 1) / spb),
                  (unsigned)((groups + kGroupsPerCta - 1) / kGroupsPerCta));
  const int ng = (int)groups;
  const uint4* s4 = static_cast<const uint4*>(src);
  uint4* d4 = static_cast<uint4*>(dst);
  const int nt = (int)n_tokens, ns = (int)n_slots;
  if (D == 128) {
    if (scatter) gather_tokens_kernel<true, 128><<<grid, 256, 0, stream>>>(s4, d4, slot_token, nt, ns, ng);
    else gather_tokens_kernel<false, 128><<<grid, 256, 0, stream>>>(s4, d4, slot_token, nt, ns, ng);
  } else if (D == 64) {
    if (scatter) gather_tokens_kernel<true, 64><<<grid, 256, 0, stream>>>(s4, d4, slot_token, nt, ns, ng);
    else gather_tokens_kernel<false, 64><<<grid, 256, 0, stream>>>(s4, d4, slot_token, nt, ns, ng);
  } else {
    const dim3 g1((unsigned)n_slots, (unsigned)groups);
    if (scatter) gather_tokens_any_kernel<true><<<g1, 256, 0, stream>>>(s4, d4, slot_token, nt, ns, D / 8);
    else gather_tokens_any_kernel<false><<<g1, 256, 0, stream>>>(s4, d4, slot_token, nt, ns, D / 8);
  }
  return cudaGetLastError() == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

}  // namespace vsa
