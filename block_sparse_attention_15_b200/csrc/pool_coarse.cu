// a1 block mean-pooling and a2+a3 coarse attention with top-k selection.
//
// Pooling ("[perf] avoid full-sequence materialization in VSA coarse/sparse
// combine", Problem / Notes: the compression branch runs on per-block means,
// taken as an fp32 block sum) is a pure HBM stream: every CTA reads one
// 64-slot block with 16-byte loads, all issued before any use, and reduces in
// fp32.  For q and k it also keeps the block's largest row norm, from which
// the coarse kernel forms a bound on every logit of a query block (the
// sparse kernel's vote-free step relies on it).  Coarse attention plus top-k ("[chore] release fastvideo-kernel
// 0.3.0", index-native q2k_idx / q2k_num) is tiny (a few GFLOP per forward);
// it keeps a tile of pooled queries and one score row per query block in
// shared memory, runs fp32 SIMT dot products, picks the top-k by a bitwise
// search for the k-th largest order-preserving integer key (ties to the lower
// index) and writes the selection in ascending order.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "vsa.h"
#include "vsa_device.cuh"
#include "vsa_launch.h"

namespace vsa {

// ---------------------------------------------------------------------------
// a1: pooling.  One CTA of 256 threads per (tensor, batch*head, block) of
// BS slots (64, 128 or 256).
// ---------------------------------------------------------------------------
template <int D, int BS>
__global__ void __launch_bounds__(256, BS == 64 ? 8 : 6) pool_kernel(PoolParams p) {
  constexpr int CPR = D / 8;          // 16-byte chunks per row
  constexpr int RPP = 256 / CPR;      // rows per pass
  constexpr int CHUNK = 64;           // rows held in registers at a time
  constexpr int PASSES = CHUNK / RPP;
  static_assert(BS % CHUNK == 0, "block must be a multiple of 64 slots");
  __shared__ float red[RPP][D + 1];
  __shared__ float wmax[8];

  // 32-bit index arithmetic: the launcher caps the grid below 2^31 CTAs
  int item = (int)blockIdx.x;
  const int nq_items = p.groups * p.nq;
  const int nkv_items = p.groups * p.nkv;
  const __nv_bfloat16* src;
  Strides3 st;
  const int32_t* bs;
  float* dst;
  float* nrm;        // largest row norm of the block, or null
  bool all_rows;     // the norm covers the padding rows too (query side)
  int nblocks;
  if (item < nq_items) {
    src = p.q; st = p.q_st; bs = p.q_bs; dst = p.qc; nblocks = p.nq; nrm = p.qn; all_rows = true;
  } else if (item < nq_items + nkv_items) {
    item -= nq_items;
    src = p.k; st = p.k_st; bs = p.kv_bs; dst = p.kc; nblocks = p.nkv; nrm = p.kn; all_rows = false;
  } else {
    item -= nq_items + nkv_items;
    src = p.v; st = p.v_st; bs = p.kv_bs; dst = p.vc; nblocks = p.nkv; nrm = nullptr; all_rows = false;
  }
  const int group = item / nblocks;
  const int blk = item - group * nblocks;
  const int b = group / p.H, h = group - b * p.H;
  int m = bs ? bs[blk] : BS;
  if (m < 1 || m > BS) {
    if (threadIdx.x == 0) set_status(p.status, VSA_ERR_BLOCK_SIZE);
    m = m < 1 ? 1 : BS;
  }
  const int lim = (nrm && all_rows) ? BS : m;  // rows read
  const int chunk = threadIdx.x % CPR;
  const int r0 = threadIdx.x / CPR;
  // contiguous [B, H, S, D]: the block is BS consecutive rows; else the
  // block's first slot in the strided view (item = group*nblocks + blk)
  const bool contiguous = st.s == D && st.h == (long long)nblocks * BS * D && st.b == st.h * p.H;
  const __nv_bfloat16* base = contiguous ? src + (long long)item * BS * D
                                         : src + b * st.b + h * st.h + (long long)BS * blk * st.s;
  const long long rstride = contiguous ? (long long)D : st.s;

  // block sums over the real rows and the largest squared row norm (over
  // every row read), 64 rows at a time with every load of a chunk issued
  // before any use
  float acc[8], mx = 0.f;
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  const uint4* rp = reinterpret_cast<const uint4*>(base + r0 * rstride) + chunk;
  const long long pstride = rstride * RPP / 8;  // uint4 units between passes
#pragma unroll 1
  for (int c0 = 0; c0 < BS; c0 += CHUNK, rp += pstride * PASSES) {
    if (c0 >= lim) break;
    uint4 buf[PASSES];
#pragma unroll
    for (int ps = 0; ps < PASSES; ++ps) {
      const int row = c0 + r0 + ps * RPP;
      buf[ps] = row < lim ? __ldcs(rp + ps * pstride) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int ps = 0; ps < PASSES; ++ps) {
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&buf[ps]);
      const bool real = c0 + r0 + ps * RPP < m;
      float sq = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(h2[e]);
        sq = fmaf(f.x, f.x, sq);
        sq = fmaf(f.y, f.y, sq);
        if (real) {
          acc[2 * e] += f.x;
          acc[2 * e + 1] += f.y;
        }
      }
      if (nrm) {
        // a row's CPR chunks sit in CPR consecutive lanes
#pragma unroll
        for (int o = CPR / 2; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
        mx = fmaxf(mx, sq);
      }
    }
  }
  if (nrm) {
#pragma unroll
    for (int o = CPR; o < 32; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = mx;
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) red[r0][chunk * 8 + e] = acc[e];
  __syncthreads();
  if (threadIdx.x < D) {
    float s = 0.f;
#pragma unroll
    for (int r = 0; r < RPP; ++r) s += red[r][threadIdx.x];
    dst[(long long)item * D + threadIdx.x] = __fdiv_rn(s, (float)m);
  }
  if (nrm && threadIdx.x == 0) {
    float mx = wmax[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) mx = fmaxf(mx, wmax[w]);
    nrm[item] = __fsqrt_rn(mx);
  }
}

// ---------------------------------------------------------------------------
// a2 + a3: coarse attention and top-k.  One CTA of 256 threads (8 warps) per
// (batch*head, tile of kQT query blocks); two CTAs per SM.
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

constexpr int kQT = 16;        // query blocks per CTA
constexpr int kCH = 64;        // pooled key / value rows per staged chunk

// Shared memory of one CTA (byte offsets; the score rows have a runtime pitch).
template <int D>
struct CoarseSmem {
  static constexpr int LD = D + 4;  // row pitch in floats: 16-byte column reads hit distinct banks
  static constexpr uint32_t kQs = 0;                                  // [kQT][LD]
  static constexpr uint32_t kCs = kQs + kQT * LD * 4;                 // [2][kCH][LD]
  static constexpr uint32_t kRowSum = kCs + 2 * kCH * LD * 4;         // [kQT]
  static constexpr uint32_t kKnMax = kRowSum + kQT * 4;               // [8] per-warp largest key norm
  static constexpr uint32_t kBars = kKnMax + 8 * 4;                   // [3] u64: two chunk buffers, query tile
  static constexpr uint32_t kSc = kBars + 32;                         // [kQT][sp] f32
  static_assert(kCs % 128 == 0 && (kCH * LD * 4) % 128 == 0, "TMA destinations");
  static uint32_t bytes(int sp) { return kSc + (uint32_t)kQT * sp * 4u; }
};

// k-th largest key of one row (n <= 32 * KPL keys in shared memory, one
// warp): the largest T with at least k keys >= T, built two bits at a time
// from the most significant, the three candidates' counts taken by the whole
// warp in independent reductions over keys held in registers; ties_needed is
// how many keys equal to T belong to the top k.  No shared-memory atomics:
// the scores of one row share their leading bits, which would pile a
// histogram's increments onto a few bins.  Padding keys are 0, below every
// finite score's key.
template <int KPL>
__device__ __forceinline__ uint32_t bitwise_select(const uint32_t* keys, int n, uint32_t k, int lane,
                                                   uint32_t& ties_needed) {
  uint32_t kr[KPL];
#pragma unroll
  for (int i = 0; i < KPL; ++i) {
    const int j = lane + 32 * i;
    kr[i] = j < n ? keys[j] : 0u;
  }
  uint32_t T = 0u;
#pragma unroll 1
  for (int b = 30; b >= 0; b -= 2) {
    const uint32_t c1 = T | (1u << b), c2 = T | (2u << b), c3 = T | (3u << b);
    uint32_t n1 = 0u, n2 = 0u, n3 = 0u;
#pragma unroll
    for (int i = 0; i < KPL; ++i) {
      n1 += kr[i] >= c1 ? 1u : 0u;
      n2 += kr[i] >= c2 ? 1u : 0u;
      n3 += kr[i] >= c3 ? 1u : 0u;
    }
    n1 = __reduce_add_sync(0xffffffffu, n1);
    n2 = __reduce_add_sync(0xffffffffu, n2);
    n3 = __reduce_add_sync(0xffffffffu, n3);
    T = n3 >= k ? c3 : n2 >= k ? c2 : n1 >= k ? c1 : T;
  }
  uint32_t above = 0u;
#pragma unroll
  for (int i = 0; i < KPL; ++i) above += kr[i] > T ? 1u : 0u;
  ties_needed = k - __reduce_add_sync(0xffffffffu, above);
  return T;
}

// The pooled tensors are read through 3D tensor maps (D, blocks, groups) whose
// boxes are D + 4 columns wide: the 4 columns past D are out of range and
// arrive as zeros, which gives the padded row pitch in one TMA request per
// chunk; rows past a group's last block arrive as zeros too.
template <int D>
__global__ void __launch_bounds__(256, 2)
    coarse_topk_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, CoarseParams p) {
  using S = CoarseSmem<D>;
  constexpr int LD = S::LD;
  constexpr int DV = D / 32;  // head dims per thread in the output product
  extern __shared__ __align__(128) uint8_t csm[];
  float* qs = reinterpret_cast<float*>(csm + S::kQs);
  float* cs = reinterpret_cast<float*>(csm + S::kCs);
  float* rowsum = reinterpret_cast<float*>(csm + S::kRowSum);
  uint64_t* bars = reinterpret_cast<uint64_t*>(csm + S::kBars);
  float* sc = reinterpret_cast<float*>(csm + S::kSc);
  const int nkv_pad = (p.nkv + kCH - 1) / kCH * kCH;
  const int sp = nkv_pad + 4;  // score row pitch: rows start on different banks
  const int nch = nkv_pad / kCH;

  const int group = blockIdx.y;
  const int a0 = blockIdx.x * kQT;
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int ty = lane / 8, tx = lane % 8;
  volatile int abort_flag_s = 0;
  volatile int* abort_flag = &abort_flag_s;

  if (tid == 0) {
    mbar_init(bars, 1);
    mbar_init(bars + 1, 1);
    mbar_init(bars + 2, 1);
    mbar_fence_init();
  }
  __syncthreads();
  // chunk stream: kc chunks 0..nch-1, then vc chunks; chunk t lands in buffer t & 1
  auto issue_chunk = [&](int t) {
    mbar_arrive_expect_tx(bars + (t & 1), (uint32_t)(kCH * LD * 4));
    tma_load_3d(cs + (t & 1) * kCH * LD, t < nch ? &tm_k : &tm_v, bars + (t & 1), 0, (t % nch) * kCH, group);
  };
  if (tid == 0) {
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    // pooled query tile (rows past nq arrive as zeros)
    mbar_arrive_expect_tx(bars + 2, (uint32_t)(kQT * LD * 4));
    tma_load_3d(qs, &tm_q, bars + 2, 0, a0, group);
    issue_chunk(0);
    issue_chunk(1);
  }
  if (p.qk_bound) {
    // largest key row norm of the group (every CTA of the group takes it)
    float km = 0.f;
    for (int j = tid; j < p.nkv; j += 256) km = fmaxf(km, p.kn[(long long)group * p.nkv + j]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) km = fmaxf(km, __shfl_xor_sync(0xffffffffu, km, o));
    if (lane == 0) reinterpret_cast<float*>(csm + S::kKnMax)[warp] = km;
  }
  warp_wait(bars + 2, 0u, abort_flag, p.status);

  // scores = scale * qc . kc: warp w owns row 8w + tx of each chunk, a
  // thread query rows ty + 4r
  for (int t = 0; t < nch; ++t) {
    // (a wait that gives up has recorded the timeout; later waits give up at once)
    warp_wait(bars + (t & 1), (uint32_t)((t >> 1) & 1), abort_flag, p.status);
    const float* cb = cs + (t & 1) * kCH * LD;
    float acc[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) acc[r] = 0.f;
#pragma unroll 8
    for (int d = 0; d < D; d += 4) {
      float4 qv[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) qv[r] = *reinterpret_cast<const float4*>(qs + (ty + 4 * r) * LD + d);
      const float4 kv = *reinterpret_cast<const float4*>(cb + (8 * warp + tx) * LD + d);
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        acc[r] = fmaf(qv[r].x, kv.x, acc[r]);
        acc[r] = fmaf(qv[r].y, kv.y, acc[r]);
        acc[r] = fmaf(qv[r].z, kv.z, acc[r]);
        acc[r] = fmaf(qv[r].w, kv.w, acc[r]);
      }
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) sc[(ty + 4 * r) * sp + t * kCH + 8 * warp + tx] = acc[r] * p.scale;
    __syncthreads();  // buffer t & 1 is free again
    if (tid == 0 && t + 2 < 2 * nch) issue_chunk(t + 2);
  }

  // logit bound per query block of the tile (the per-warp key norms were
  // published before the score loop's barriers)
  if (p.qk_bound && tid < kQT && a0 + tid < p.nq) {
    const float* kw = reinterpret_cast<const float*>(csm + S::kKnMax);
    float km = kw[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) km = fmaxf(km, kw[w]);
    const long long qi = (long long)group * p.nq + a0 + tid;
    p.qk_bound[qi] = p.bound_scale * p.qn[qi] * km;
  }

  // per row: top-k on the scaled logits, then the softmax numerators
  const int k = p.topk;  // already clamped to [1, nkv]
  for (int r = warp; r < kQT; r += 8) {
    const int a = a0 + r;
    float* row = sc + r * sp;
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
    __syncwarp();
    uint32_t ties_needed;
    uint32_t T;
    if (p.nkv <= 256) T = bitwise_select<8>(keys, p.nkv, (uint32_t)k, lane, ties_needed);
    else if (p.nkv <= 512) T = bitwise_select<16>(keys, p.nkv, (uint32_t)k, lane, ties_needed);
    else if (p.nkv <= 1024) T = bitwise_select<32>(keys, p.nkv, (uint32_t)k, lane, ties_needed);
    else T = bitwise_select<64>(keys, p.nkv, (uint32_t)k, lane, ties_needed);
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

  // out_c = (e . vc) / rowsum: warp w owns a quarter of the head dims (DV
  // consecutive ones per thread) for query rows 8 (w / 4) + ty + 4r, r < 2
  const int d0 = (warp % 4) * (D / 4) + tx * DV;
  const int qr0 = 8 * (warp / 4) + ty;
  float acc[2][DV];
#pragma unroll
  for (int r = 0; r < 2; ++r)
#pragma unroll
    for (int e = 0; e < DV; ++e) acc[r][e] = 0.f;
  for (int t = nch; t < 2 * nch; ++t) {
    // (a wait that gives up has recorded the timeout; later waits give up at once)
    warp_wait(bars + (t & 1), (uint32_t)((t >> 1) & 1), abort_flag, p.status);
    const float* cb = cs + (t & 1) * kCH * LD;
    const int c0 = (t - nch) * kCH;
#pragma unroll 2
    for (int c = 0; c < kCH; c += 4) {
      float4 ev[2];
#pragma unroll
      for (int r = 0; r < 2; ++r) ev[r] = *reinterpret_cast<const float4*>(sc + (qr0 + 4 * r) * sp + c0 + c);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        float vv[DV];
        if constexpr (DV == 4) {
          const float4 v4 = *reinterpret_cast<const float4*>(cb + (c + u) * LD + d0);
          vv[0] = v4.x; vv[1] = v4.y; vv[2] = v4.z; vv[3] = v4.w;
        } else {
          const float2 v2 = *reinterpret_cast<const float2*>(cb + (c + u) * LD + d0);
          vv[0] = v2.x; vv[1] = v2.y;
        }
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const float pr = u == 0 ? ev[r].x : u == 1 ? ev[r].y : u == 2 ? ev[r].z : ev[r].w;
#pragma unroll
          for (int e = 0; e < DV; ++e) acc[r][e] = fmaf(pr, vv[e], acc[r][e]);
        }
      }
    }
    __syncthreads();
    if (tid == 0 && t + 2 < 2 * nch) issue_chunk(t + 2);
  }
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int a = a0 + qr0 + 4 * r;
    if (a >= p.nq) continue;
    const float inv = 1.f / rowsum[qr0 + 4 * r];
    float* dst = p.out_c + ((long long)group * p.nq + a) * D + d0;
    if constexpr (DV == 4) {
      *reinterpret_cast<float4*>(dst) = make_float4(acc[r][0] * inv, acc[r][1] * inv, acc[r][2] * inv, acc[r][3] * inv);
    } else {
      *reinterpret_cast<float2*>(dst) = make_float2(acc[r][0] * inv, acc[r][1] * inv);
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
  if (p.block == 256) {
    if (D == 128) pool_kernel<128, 256><<<(unsigned)items, 256, 0, stream>>>(p);
    else pool_kernel<64, 256><<<(unsigned)items, 256, 0, stream>>>(p);
  } else if (p.block == 128) {
    if (D == 128) pool_kernel<128, 128><<<(unsigned)items, 256, 0, stream>>>(p);
    else pool_kernel<64, 128><<<(unsigned)items, 256, 0, stream>>>(p);
  } else {
    if (D == 128) pool_kernel<128, 64><<<(unsigned)items, 256, 0, stream>>>(p);
    else pool_kernel<64, 64><<<(unsigned)items, 256, 0, stream>>>(p);
  }
  return cudaGetLastError() == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

// 3D fp32 map (D, n, groups) over a [groups][n][D] array, boxes of
// (D + 4) x rows x 1 (the 4 extra columns are out of range: zeros).
static bool make_pooled_map(CUtensorMap* map, const float* base, int D, int n, int groups, int rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)n, (cuuint64_t)groups};
  cuuint64_t strides[2] = {(cuuint64_t)D * 4, (cuuint64_t)n * D * 4};
  cuuint32_t box[3] = {(cuuint32_t)(D + 4), (cuuint32_t)rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
static int launch_coarse_t(const CoarseParams& p, cudaStream_t stream) {
  const int nkv_pad = (p.nkv + kCH - 1) / kCH * kCH;
  const size_t smem = CoarseSmem<D>::bytes(nkv_pad + 4);
  if (smem > 227 * 1024) return VSA_ERR_UNSUPPORTED;
  CUtensorMap mq, mk, mv;
  if (!make_pooled_map(&mq, p.qc, D, p.nq, p.groups, kQT) || !make_pooled_map(&mk, p.kc, D, p.nkv, p.groups, kCH) ||
      !make_pooled_map(&mv, p.vc, D, p.nkv, p.groups, kCH))
    return VSA_ERR_CUDA;
  auto kern = coarse_topk_kernel<D>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return VSA_ERR_CUDA;
  dim3 grid((p.nq + kQT - 1) / kQT, p.groups);
  kern<<<grid, 256, smem, stream>>>(mq, mk, mv, p);
  return cudaGetLastError() == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

int launch_coarse_topk(const CoarseParams& p, int D, cudaStream_t stream) {
  return D == 128 ? launch_coarse_t<128>(p, stream) : launch_coarse_t<64>(p, stream);
}

}  // namespace vsa
