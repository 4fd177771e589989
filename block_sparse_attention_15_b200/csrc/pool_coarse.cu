// a1 block mean-pooling and a2+a3 coarse attention with top-k selection.
//
// Pooling ("[perf] avoid full-sequence materialization in VSA coarse/sparse
// combine", Problem / Notes: the compression branch runs on per-block means,
// taken as an fp32 block sum) is a pure HBM stream: every CTA reads one
// 64-slot block with 16-byte loads, all issued before any use, and reduces in
// fp32.  Coarse attention plus top-k ("[chore] release fastvideo-kernel
// 0.3.0", index-native q2k_idx / q2k_num) is tiny (a few GFLOP per forward);
// it keeps a tile of pooled queries and one score row per query block in
// shared memory, runs fp32 SIMT dot products, picks the top-k by a bitwise
// radix select on order-preserving integer keys (ties to the lower index)
// and writes the selection in ascending order.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "vsa.h"
#include "vsa_device.cuh"
#include "vsa_launch.h"

namespace vsa {

// ---------------------------------------------------------------------------
// a1: pooling.  One CTA of 256 threads per (tensor, batch*head, block).
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) pool_kernel(PoolParams p) {
  constexpr int CPR = D / 8;          // 16-byte chunks per row
  constexpr int RPP = 256 / CPR;      // rows per pass
  constexpr int PASSES = 64 / RPP;
  __shared__ float red[RPP][D + 1];

  long long item = blockIdx.x;
  const long long nq_items = (long long)p.groups * p.nq;
  const long long nkv_items = (long long)p.groups * p.nkv;
  const __nv_bfloat16* src;
  const int32_t* bs;
  float* dst;
  int nblocks;
  if (item < nq_items) {
    src = p.q; bs = p.q_bs; dst = p.qc; nblocks = p.nq;
  } else if (item < nq_items + nkv_items) {
    item -= nq_items;
    src = p.k; bs = p.kv_bs; dst = p.kc; nblocks = p.nkv;
  } else {
    item -= nq_items + nkv_items;
    src = p.v; bs = p.kv_bs; dst = p.vc; nblocks = p.nkv;
  }
  const int blk = (int)(item % nblocks);
  int m = bs ? bs[blk] : 64;
  if (m < 1 || m > 64) {
    if (threadIdx.x == 0) set_status(p.status, VSA_ERR_BLOCK_SIZE);
    m = m < 1 ? 1 : 64;
  }
  const __nv_bfloat16* base = src + item * 64 * D;  // item = group*nblocks + blk
  const int chunk = threadIdx.x % CPR;
  const int r0 = threadIdx.x / CPR;

  uint4 buf[PASSES];
#pragma unroll
  for (int ps = 0; ps < PASSES; ++ps) {
    const int row = r0 + ps * RPP;
    if (row < m) {
      buf[ps] = __ldcs(reinterpret_cast<const uint4*>(base + (long long)row * D) + chunk);
    } else {
      buf[ps] = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
  for (int ps = 0; ps < PASSES; ++ps) {
    const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&buf[ps]);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float2 f = __bfloat1622float2(h2[e]);
      acc[2 * e] += f.x;
      acc[2 * e + 1] += f.y;
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) red[r0][chunk * 8 + e] = acc[e];
  __syncthreads();
  if (threadIdx.x < D) {
    float s = 0.f;
#pragma unroll
    for (int r = 0; r < RPP; ++r) s += red[r][threadIdx.x];
    dst[item * D + threadIdx.x] = __fdiv_rn(s, (float)m);
  }
}

// ---------------------------------------------------------------------------
// a2 + a3: coarse attention and top-k.  One CTA of 256 threads per
// (batch*head, tile of QT query blocks).
// ---------------------------------------------------------------------------
// Order-preserving map from fp32 to uint32 (larger float -> larger key).
__device__ __forceinline__ uint32_t float_to_key(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_to_float(uint32_t k) {
  uint32_t u = (k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k;
  return __uint_as_float(u);
}

template <int D, int QT>
__global__ void __launch_bounds__(256) coarse_topk_kernel(CoarseParams p) {
  constexpr int LD = D + 4;           // padded row pitch (floats), keeps float4 alignment
  constexpr int RT = QT / 16;         // query rows per thread in the score product
  extern __shared__ __align__(16) float smem[];
  float* qs = smem;                   // [QT][LD]
  float* cs = qs + QT * LD;           // [64][LD]   kc or vc chunk
  float* rowsum = cs + 64 * LD;       // [QT]
  float* sc = rowsum + QT;            // [QT][nkv_pad]
  const int nkv_pad = (p.nkv + 63) & ~63;

  const int group = blockIdx.y;
  const int a0 = blockIdx.x * QT;
  const int tid = threadIdx.x;
  const int ty = tid / 16, tx = tid % 16;
  const float* qc = p.qc + (long long)group * p.nq * D;
  const float* kc = p.kc + (long long)group * p.nkv * D;
  const float* vc = p.vc + (long long)group * p.nkv * D;

  // pooled query tile
  for (int i = tid; i < QT * (D / 4); i += 256) {
    const int r = i / (D / 4), c4 = i % (D / 4);
    float4 val = make_float4(0.f, 0.f, 0.f, 0.f);
    if (a0 + r < p.nq) val = reinterpret_cast<const float4*>(qc + (long long)(a0 + r) * D)[c4];
    *reinterpret_cast<float4*>(qs + r * LD + 4 * c4) = val;
  }

  // scores = scale * qc . kc, one 64-block chunk of kc at a time
  for (int c0 = 0; c0 < nkv_pad; c0 += 64) {
    __syncthreads();
    for (int i = tid; i < 64 * (D / 4); i += 256) {
      const int r = i / (D / 4), c4 = i % (D / 4);
      float4 val = make_float4(0.f, 0.f, 0.f, 0.f);
      if (c0 + r < p.nkv) val = reinterpret_cast<const float4*>(kc + (long long)(c0 + r) * D)[c4];
      *reinterpret_cast<float4*>(cs + r * LD + 4 * c4) = val;
    }
    __syncthreads();
    float acc[RT][4];
#pragma unroll
    for (int r = 0; r < RT; ++r)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[r][i] = 0.f;
#pragma unroll 4
    for (int d = 0; d < D; d += 4) {
      float4 qv[RT], kv[4];
#pragma unroll
      for (int r = 0; r < RT; ++r) qv[r] = *reinterpret_cast<const float4*>(qs + (ty * RT + r) * LD + d);
#pragma unroll
      for (int i = 0; i < 4; ++i) kv[i] = *reinterpret_cast<const float4*>(cs + (tx + 16 * i) * LD + d);
#pragma unroll
      for (int r = 0; r < RT; ++r)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc[r][i] = fmaf(qv[r].x, kv[i].x, acc[r][i]);
          acc[r][i] = fmaf(qv[r].y, kv[i].y, acc[r][i]);
          acc[r][i] = fmaf(qv[r].z, kv[i].z, acc[r][i]);
          acc[r][i] = fmaf(qv[r].w, kv[i].w, acc[r][i]);
        }
    }
#pragma unroll
    for (int r = 0; r < RT; ++r)
#pragma unroll
      for (int i = 0; i < 4; ++i) sc[(ty * RT + r) * nkv_pad + c0 + tx + 16 * i] = acc[r][i] * p.scale;
  }
  __syncthreads();

  // per row: top-k on the scaled logits, then the softmax numerators
  const int warp = tid / 32, lane = tid % 32;
  const int k = p.topk;  // already clamped to [1, nkv]
  for (int r = warp; r < QT; r += 8) {
    const int a = a0 + r;
    float* row = sc + r * nkv_pad;
    if (a >= p.nq) {
      for (int j = lane; j < nkv_pad; j += 32) row[j] = 0.f;
      if (lane == 0) rowsum[r] = 1.f;
      continue;
    }
    uint32_t* keys = reinterpret_cast<uint32_t*>(row);
    uint32_t kmax = 0u;
    for (int j = lane; j < p.nkv; j += 32) {
      const uint32_t kk = float_to_key(row[j]);
      keys[j] = kk;
      kmax = max(kmax, kk);
    }
    kmax = __reduce_max_sync(0xffffffffu, kmax);
    // largest T with #{key >= T} >= k: the k-th largest key
    uint32_t T = 0u;
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t cand = T | (1u << bit);
      uint32_t cnt = 0u;
      for (int j = lane; j < p.nkv; j += 32) cnt += (keys[j] >= cand) ? 1u : 0u;
      cnt = __reduce_add_sync(0xffffffffu, cnt);
      if (cnt >= (uint32_t)k) T = cand;
    }
    uint32_t gt = 0u;
    for (int j = lane; j < p.nkv; j += 32) gt += (keys[j] > T) ? 1u : 0u;
    gt = __reduce_add_sync(0xffffffffu, gt);
    const uint32_t ties_needed = (uint32_t)k - gt;
    // ascending compaction: keys above T, then the lowest-index ties
    int32_t* out_idx = p.q2k_idx + ((long long)group * p.nq + a) * p.idx_stride;
    uint32_t written = 0u, ties_seen = 0u;
    for (int j0 = 0; j0 < p.nkv; j0 += 32) {
      const int j = j0 + lane;
      const uint32_t kk = (j < p.nkv) ? keys[j] : 0u;
      const bool above = (j < p.nkv) && kk > T;
      const bool tie = (j < p.nkv) && kk == T;
      const uint32_t tie_mask = __ballot_sync(0xffffffffu, tie);
      const uint32_t tie_rank = ties_seen + __popc(tie_mask & ((1u << lane) - 1u));
      const bool sel = above || (tie && tie_rank < ties_needed);
      const uint32_t sel_mask = __ballot_sync(0xffffffffu, sel);
      if (sel) out_idx[written + __popc(sel_mask & ((1u << lane) - 1u))] = j;
      written += __popc(sel_mask);
      ties_seen += __popc(tie_mask);
    }
    for (int j = k + lane; j < p.idx_stride; j += 32) out_idx[j] = -1;
    if (lane == 0) p.q2k_num[(long long)group * p.nq + a] = k;
    // softmax numerators exp(s - max) in place, padded columns 0
    const float m = key_to_float(kmax);
    float sum = 0.f;
    for (int j = lane; j < nkv_pad; j += 32) {
      float e = 0.f;
      if (j < p.nkv) e = expf(key_to_float(keys[j]) - m);
      row[j] = e;
      sum += e;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane == 0) rowsum[r] = sum;
  }
  __syncthreads();

  // out_c = (e . vc) / rowsum; thread columns tx*4 + 64*j, rows ty*RT + r
  constexpr int CJ = D / 64;
  float acc[RT][CJ][4];
#pragma unroll
  for (int r = 0; r < RT; ++r)
#pragma unroll
    for (int j = 0; j < CJ; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[r][j][e] = 0.f;
  for (int c0 = 0; c0 < nkv_pad; c0 += 64) {
    for (int i = tid; i < 64 * (D / 4); i += 256) {
      const int r = i / (D / 4), c4 = i % (D / 4);
      float4 val = make_float4(0.f, 0.f, 0.f, 0.f);
      if (c0 + r < p.nkv) val = reinterpret_cast<const float4*>(vc + (long long)(c0 + r) * D)[c4];
      *reinterpret_cast<float4*>(cs + r * LD + 4 * c4) = val;
    }
    __syncthreads();
#pragma unroll 4
    for (int c = 0; c < 64; ++c) {
      float pr[RT];
#pragma unroll
      for (int r = 0; r < RT; ++r) pr[r] = sc[(ty * RT + r) * nkv_pad + c0 + c];
#pragma unroll
      for (int j = 0; j < CJ; ++j) {
        const float4 vv = *reinterpret_cast<const float4*>(cs + c * LD + 64 * j + 4 * tx);
#pragma unroll
        for (int r = 0; r < RT; ++r) {
          acc[r][j][0] = fmaf(pr[r], vv.x, acc[r][j][0]);
          acc[r][j][1] = fmaf(pr[r], vv.y, acc[r][j][1]);
          acc[r][j][2] = fmaf(pr[r], vv.z, acc[r][j][2]);
          acc[r][j][3] = fmaf(pr[r], vv.w, acc[r][j][3]);
        }
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int r = 0; r < RT; ++r) {
    const int a = a0 + ty * RT + r;
    if (a >= p.nq) continue;
    const float inv = 1.f / rowsum[ty * RT + r];
#pragma unroll
    for (int j = 0; j < CJ; ++j) {
      float4 o = make_float4(acc[r][j][0] * inv, acc[r][j][1] * inv, acc[r][j][2] * inv,
                             acc[r][j][3] * inv);
      *reinterpret_cast<float4*>(p.out_c + ((long long)group * p.nq + a) * D + 64 * j + 4 * tx) = o;
    }
  }
}

// ---------------------------------------------------------------------------
// host launchers
// ---------------------------------------------------------------------------
int launch_pool(const PoolParams& p, int D, cudaStream_t stream) {
  const long long items = (long long)p.groups * (p.nq + 2LL * p.nkv);
  if (items <= 0) return VSA_OK;
  if (items > 0x7FFFFFFFLL) return VSA_ERR_UNSUPPORTED;
  if (D == 128) pool_kernel<128><<<(unsigned)items, 256, 0, stream>>>(p);
  else pool_kernel<64><<<(unsigned)items, 256, 0, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

template <int D, int QT>
static int launch_coarse_t(const CoarseParams& p, cudaStream_t stream) {
  const int nkv_pad = (p.nkv + 63) & ~63;
  const size_t smem = sizeof(float) * ((size_t)(QT + 64) * (D + 4) + QT + (size_t)QT * nkv_pad);
  if (smem > 227 * 1024) return VSA_ERR_UNSUPPORTED;
  auto kern = coarse_topk_kernel<D, QT>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return VSA_ERR_CUDA;
  dim3 grid((p.nq + QT - 1) / QT, p.groups);
  kern<<<grid, 256, smem, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

int launch_coarse_topk(const CoarseParams& p, int D, cudaStream_t stream) {
  if (p.nkv <= 1280) {
    return D == 128 ? launch_coarse_t<128, 32>(p, stream) : launch_coarse_t<64, 32>(p, stream);
  }
  return D == 128 ? launch_coarse_t<128, 16>(p, stream) : launch_coarse_t<64, 16>(p, stream);
}

}  // namespace vsa
