// Backward of the block-sparse attention over selected 64 x 64 tiles:
// dq, dk, dv from the output gradient, the forward's output and its
// per-row log-sum-exp.
//
// What it computes ("[kernel] Add varlen support for block-sparse attention",
// Summary / Backward correctness: dQ/dK/dV of the block-sparse attention,
// and a varlen backward through a k2q, KV block -> query blocks, index):
// with P = softmax(scale * q k^T) over each query block's selected keys,
//   delta_i = sum_d dout_i * out_i,   dS = P * (dout v^T - delta),
//   dq = scale * dS k,  dk = scale * dS^T q,  dv = P^T dout.
//
// How (sm_100a), three passes:
//  * delta: one row per 16 threads, fp32 sums;
//  * dq: query-block-stationary, the forward's transposed pair-of-tiles
//    formulation: per pair of selected KV tiles (M = 128 key rows)
//      S^T = K2 . Q^T,  dP^T = V2 . dO^T             (into TMEM)
//      dS^T = P^T * (dP^T - delta)                     (softmax warps, smem, bf16)
//      dQ^T += K2^T . dS^T                             (TMEM, M = head dim)
//  * dk/dv: KV-block-stationary over the k2q index, two query blocks per
//    step (M = 128 query rows, a block listed m times weighs m times):
//      S = Q2 . K^T,  dP = dO2 . V^T                   (into TMEM)
//      P, dS                                           (softmax warps, smem, bf16)
//      dV^T += dO2^T . P,  dK^T += Q2^T . dS           (TMEM, M = head dim)
// Both kernels: persistent grid of one CTA per SM, warp-specialised (load
// warp, MMA warp, two compute warpgroups splitting the 64 columns, epilogue
// warpgroup), bounded waits, TMA loads through the same 4-D maps of strided
// views as the forward (no multicast).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "vsa.h"
#include "vsa_device.cuh"
#include "vsa_launch.h"

namespace vsa {
namespace bwd {

constexpr int kThreads = 512;
constexpr uint32_t kRegsProducer = 64, kRegsCompute = 192, kRegsEpilogue = 64;
static_assert(128u * (kRegsProducer + 2u * kRegsCompute + kRegsEpilogue) <= 512u * 128u,
              "register split exceeds the launch's 128 registers per thread");

// A pair of 64-row tiles: [dh][2 tiles][64 rows][128 B]; a single tile:
// [dh][64 rows][128 B] (128-byte swizzle, 1 KB atoms).
__device__ __forceinline__ uint32_t pair_off(int dh, int tile) {
  return uint32_t(dh) * 16384u + uint32_t(tile) * 8192u;
}

// D[128][64] = A[128][D] . B[64][D]^T, A a pair (K-major), B a single tile
// (K-major).
template <int D>
__device__ __forceinline__ void mma_pair_single(uint32_t tmem_d, uint32_t a_base, uint32_t b_base) {
  constexpr uint32_t idesc = make_idesc_bf16(128, 64, false, false);
  const uint64_t a0 = make_sdesc_sw128(a_base, 16u, 1024u);
  const uint64_t b0 = make_sdesc_sw128(b_base, 16u, 1024u);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint64_t a = a0 + (uint64_t)((pair_off(kk / 4, 0) + (kk % 4) * 32) >> 4);
    const uint64_t b = b0 + (uint64_t)(((kk / 4) * 8192 + (kk % 4) * 32) >> 4);
    umma_bf16(tmem_d, a, b, idesc, kk > 0 ? 1u : 0u);
  }
}

// D[D][64] (+)= A^T . B with A a pair [128 rows][D] read MN-major (M = head
// dim, K = the pair's 128 rows) and B [128 rows][64] MN-major in shared
// memory.  For D = 64 the second 64-row atom of the M = 128 operand is other,
// in-bounds shared memory; TMEM lanes 64..127 then hold values no one reads.
template <int D>
__device__ __forceinline__ void mma_pairT_mn(uint32_t tmem_d, uint32_t a_base, uint32_t b_base,
                                             bool accumulate) {
  constexpr uint32_t idesc = make_idesc_bf16(128, 64, true, true);
  const uint64_t a0 = make_sdesc_sw128(a_base, D == 128 ? 16384u : 8192u, 1024u);
  const uint64_t b0 = make_sdesc_sw128(b_base, 8192u, 1024u);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    umma_bf16(tmem_d, a0 + (uint64_t)((kk * 2048) >> 4), b0 + (uint64_t)((kk * 2048) >> 4), idesc,
              (accumulate || kk > 0) ? 1u : 0u);
  }
}

__device__ __forceinline__ uint32_t sw128(uint32_t row, uint32_t chunk) {
  return row * 128u + ((chunk ^ (row & 7u)) << 4);
}

__device__ __forceinline__ void load_tile64(void* dst, const CUtensorMap* map, TmaAxes ax,
                                            uint64_t* bar, int d0, int s, int h, int b) {
  const int c1 = ax.s == 1 ? s : (ax.h == 1 ? h : b);
  const int c2 = ax.s == 2 ? s : (ax.h == 2 ? h : b);
  const int c3 = ax.s == 3 ? s : (ax.h == 3 ? h : b);
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(d0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

// --------------------------------------------------------------------------
// delta_i = sum_d dout_i * out_i (fp32), every row of [rows, D]
// --------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) delta_kernel(const __nv_bfloat16* out, Strides3 out_st,
                                                    const __nv_bfloat16* dout, Strides3 dout_st,
                                                    int H, long long S, long long rows, float* delta) {
  constexpr int CPR = D / 8;  // 16-byte chunks per row
  const long long r = ((long long)blockIdx.x * 256 + threadIdx.x) / CPR;
  const int ch = threadIdx.x % CPR;
  float acc = 0.f;
  if (r < rows) {
    const long long s = r % S, g = r / S;
    const long long b = g / H, h = g % H;
    const uint4 o4 = *reinterpret_cast<const uint4*>(out + b * out_st.b + h * out_st.h + s * out_st.s + 8 * ch);
    const uint4 d4 = *reinterpret_cast<const uint4*>(dout + b * dout_st.b + h * dout_st.h + s * dout_st.s + 8 * ch);
    const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&o4);
    const __nv_bfloat162* d2 = reinterpret_cast<const __nv_bfloat162*>(&d4);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 a = __bfloat1622float2(o2[e]), c = __bfloat1622float2(d2[e]);
      acc = fmaf(a.x, c.x, acc);
      acc = fmaf(a.y, c.y, acc);
    }
  }
#pragma unroll
  for (int o = CPR / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (r < rows && ch == 0) delta[r] = acc;
}

// --------------------------------------------------------------------------
// k2q: for every (group, KV block c) the query blocks listing c, ascending,
// packed as a | (multiplicity << 16); one warp per c.  The group's index rows
// are staged in shared memory when they fit (STAGED), else read from global
// memory.  Entries outside their sequence's KV blocks are skipped, as the
// forward skips them.
// --------------------------------------------------------------------------
template <bool STAGED>
__global__ void __launch_bounds__(256) k2q_kernel(const int32_t* q2k_idx, const int32_t* q2k_num,
                                                  int nq, int nkv, int idx_stride,
                                                  const int32_t* q_kv_base,
                                                  const int32_t* q_kv_count, int32_t* k2q,
                                                  int32_t* k2q_num) {
  extern __shared__ int32_t rows_s[];  // [nq][idx_stride], then [nq] counts
  const long long group = blockIdx.y;
  const int32_t* src = q2k_idx + group * (long long)nq * idx_stride;
  const int32_t* rows = STAGED ? rows_s : src;
  if (STAGED) {
    for (long long i = threadIdx.x; i < (long long)nq * idx_stride; i += 256) rows_s[i] = src[i];
    __syncthreads();
  }
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  for (int c = blockIdx.x * 8 + warp; c < nkv && c < (int)(blockIdx.x + 1) * 8; c += 8) {
    int32_t* out = k2q + (group * nkv + c) * (long long)nq;
    int count = 0;
    for (int a = 0; a < nq; ++a) {
      int n = q2k_num[group * nq + a];
      n = n < 0 ? 0 : (n > idx_stride ? idx_stride : n);
      const int base = q_kv_base ? q_kv_base[a] : 0;  // local -> global block numbers
      const int cnt = q_kv_count ? q_kv_count[a] : nkv;
      const int lc = c - base;                         // c as a local index of a's sequence
      int m = 0;
      if (lc >= 0 && lc < cnt)
        for (int j = lane; j < n; j += 32) m += (rows[(long long)a * idx_stride + j] == lc) ? 1 : 0;
      m = __reduce_add_sync(0xffffffffu, m);
      if (m > 0) {
        if (lane == 0) out[count] = a | (m << 16);
        ++count;
      }
    }
    if (lane == 0) k2q_num[group * nkv + c] = count;
  }
}

// --------------------------------------------------------------------------
// dq kernel
// --------------------------------------------------------------------------
// K pairs stay in shared memory until the dQ product of their pair (late);
// V pairs only until the dP product (early).  So the K ring is one stage
// deeper than the V ring, and each ring has its own barriers.
constexpr int kDqNK = 3, kDqNV = 2;

template <int D>
struct DqLayout {
  static constexpr uint32_t kTile = 64u * D * 2u;   // one 64-row tile
  static constexpr uint32_t kPair = 2u * kTile;
  static constexpr uint32_t kQOff = 0;              // Q tile
  static constexpr uint32_t kDOOff = kQOff + kTile; // dO tile
  static constexpr uint32_t kKOff = kDOOff + kTile; // [kDqNK] K pairs
  static constexpr uint32_t kVOff = kKOff + kDqNK * kPair;  // [kDqNV] V pairs
  static constexpr uint32_t kSOff = kVOff + kDqNV * kPair;  // [2] dS^T [128][64] bf16
  static constexpr uint32_t kMetaOff = kSOff + 2u * 16384u;  // [kDqNK] int2 key counts per K stage
  static constexpr uint32_t kSMetaOff = kMetaOff + 32u;      // [2] int2 per TMEM buffer
  static constexpr uint32_t kBarOff = kSMetaOff + 16u;
  static constexpr int kQFull = 0, kQEmpty = 1, kKFull = 2, kKEmpty = kKFull + kDqNK,
                       kVFull = kKEmpty + kDqNK, kVEmpty = kVFull + kDqNV,
                       kSPFull = kVEmpty + kDqNV, kSPEmpty = kSPFull + 2, kDSFull = kSPEmpty + 2,
                       kDSEmpty = kDSFull + 2, kOFull = kDSEmpty + 2, kOEmpty = kOFull + 2,
                       kNumBars = kOEmpty + 2;
  static constexpr uint32_t kMiscOff = kBarOff + 8u * kNumBars;
  static constexpr uint32_t kAlloc = kMiscOff + 16u + 1024u;
  static_assert(kKOff % 1024 == 0 && kSOff % 1024 == 0, "1 KB atoms");
  static_assert(kAlloc <= 227u * 1024u, "shared memory");
};

// Epilogue helper: this thread holds column d of a transposed accumulator
// (TMEM lane d, 16 consecutive rows q0 .. q0+15 of the output in v[]).  Lane
// pairs swap values so that each lane writes one 4-byte word (two adjacent
// head dims of one row) per two rows: a warp's stores of one row cover 64
// consecutive bytes.  Rows at or past `len` are written as 0 unless `skip_pad`.
__device__ __forceinline__ void store_cols_t(__nv_bfloat16* col_d_row0, long long row_stride,
                                             const float (&v)[16], int q0, int len, bool skip_pad,
                                             int lane) {
  const bool odd = lane & 1;
#pragma unroll
  for (int j = 0; j < 16; j += 2) {
    const float send = odd ? v[j] : v[j + 1];
    const float recv = __shfl_xor_sync(0xffffffffu, send, 1);
    // even lane: row j, head dims (d, d + 1); odd lane: row j + 1, (d - 1, d)
    const int q = q0 + j + (odd ? 1 : 0);
    const uint32_t word = odd ? pack_bf16x2(recv, v[j + 1]) : pack_bf16x2(v[j], recv);
    __nv_bfloat16* dst = col_d_row0 + (long long)q * row_stride - (odd ? 1 : 0);
    if (q < len)
      *reinterpret_cast<uint32_t*>(dst) = word;
    else if (!skip_pad)
      *reinterpret_cast<uint32_t*>(dst) = 0u;
  }
}

struct BwdItem {
  int a, h, b;
  long long group;
  int num, q_len;
  long long q_tok;
  int kv_base, kv_count;
};

__device__ __forceinline__ BwdItem load_q_item(const BwdParams& p, long long it) {
  BwdItem x;
  x.a = (int)(it % p.nq);
  const long long t = it / p.nq;
  x.h = (int)(t % p.H);
  x.b = (int)(t / p.H);
  x.group = t;
  const int num = p.q2k_num[t * p.nq + x.a];
  x.num = num < 0 ? 0 : (num > p.idx_stride ? p.idx_stride : num);
  x.q_tok = p.q_tok ? (long long)p.q_tok[x.a] : 64LL * x.a;
  const int ql = p.q_bs ? p.q_bs[x.a] : 64;
  x.q_len = ql < 1 ? 0 : (ql > 64 ? 64 : ql);
  x.kv_base = p.q_kv_base ? p.q_kv_base[x.a] : 0;
  x.kv_count = p.q_kv_count ? p.q_kv_count[x.a] : p.nkv;
  return x;
}

// first slot and real length of entry j of an item's selection (len 0 for an
// invalid entry, which is skipped)
__device__ __forceinline__ void resolve_kv(const BwdParams& p, const BwdItem& x, int j, int& row, int& len) {
  row = 0;
  len = 0;
  if (j >= x.num) return;
  const int c = p.q2k_idx[(x.group * p.nq + x.a) * (long long)p.idx_stride + j];
  if (c < 0 || c >= x.kv_count) {
    set_status(p.status, VSA_ERR_INDEX_RANGE);
    return;
  }
  const int cg = c + x.kv_base;
  row = p.kv_tok ? p.kv_tok[cg] : 64 * cg;
  len = p.kv_bs ? p.kv_bs[cg] : 64;
  if (len < 1 || len > 64) len = 0;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
              const BwdParams p) {
  using L = DqLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  int2* meta = reinterpret_cast<int2*>(smem + L::kMetaOff);
  int2* smeta = reinterpret_cast<int2*>(smem + L::kSMetaOff);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const long long n_items = (long long)p.B * p.H * p.nq;
  const long long it0 = blockIdx.x, it_step = gridDim.x;

  if (tid == 0) {
    for (int i = 0; i < L::kNumBars; ++i) {
      uint32_t count = 1;
      if (i == L::kSPEmpty || i == L::kSPEmpty + 1 || i == L::kDSFull || i == L::kDSFull + 1)
        count = 8;  // one arrival per compute warp
      if (i == L::kOEmpty || i == L::kOEmpty + 1) count = 4;   // epilogue warps
      if (i == L::kSPFull || i == L::kSPFull + 1) count = 2;   // commit + key-count record
      mbar_init(bars + i, count);
    }
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_do);
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  // TMEM: S^T buffers at 0, 64; dP^T at 128, 192; dQ^T at 256, 320

  if (warp < 4) {
    regs_dec<kRegsProducer>();
    if (warp == 0) {
      // ===================== loads =====================
      uint32_t g = 0, n = 0;
      bool ok = true;
      for (long long it = it0; ok && it < n_items; it += it_step, ++n) {
        const BwdItem x = load_q_item(p, it);
        if (lane == 0) {
          if (n >= 1) ok = mbar_wait(bars + L::kQEmpty, (n - 1) & 1, abort_flag, p.status);
          if (ok) {
            mbar_arrive_expect_tx(bars + L::kQFull, 2 * L::kTile);
#pragma unroll
            for (int dh = 0; dh < D / 64; ++dh) {
              load_tile64(smem + L::kQOff + dh * 8192, &tm_q, p.q_ax, bars + L::kQFull, dh * 64, (int)x.q_tok, x.h, x.b);
              load_tile64(smem + L::kDOOff + dh * 8192, &tm_do, p.do_ax, bars + L::kQFull, dh * 64, (int)x.q_tok, x.h, x.b);
            }
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        const int np = (x.num + 1) / 2;
        for (int i = 0; ok && i < np; ++i, ++g) {
          if (lane == 0) {
            const int ks = (int)(g % kDqNK), vs = (int)(g % kDqNV);
            const uint32_t ku = g / kDqNK, vu = g / kDqNV;
            if (ku >= 1) ok = mbar_wait(bars + L::kKEmpty + ks, (ku - 1) & 1, abort_flag, p.status);
            if (ok && vu >= 1) ok = mbar_wait(bars + L::kVEmpty + vs, (vu - 1) & 1, abort_flag, p.status);
            if (ok) {
              int r0, l0, r1, l1;
              resolve_kv(p, x, 2 * i, r0, l0);
              resolve_kv(p, x, 2 * i + 1, r1, l1);
              if (2 * i + 1 >= x.num) { r1 = r0; l1 = 0; }
              meta[ks] = make_int2(l0, l1);
              uint64_t* kfull = bars + L::kKFull + ks;
              uint64_t* vfull = bars + L::kVFull + vs;
              mbar_arrive_expect_tx(kfull, L::kPair);
              mbar_arrive_expect_tx(vfull, L::kPair);
              uint8_t* kd = smem + L::kKOff + ks * L::kPair;
              uint8_t* vd = smem + L::kVOff + vs * L::kPair;
#pragma unroll
              for (int dh = 0; dh < D / 64; ++dh) {
                load_tile64(kd + pair_off(dh, 0), &tm_k, p.k_ax, kfull, dh * 64, r0, x.h, x.b);
                load_tile64(kd + pair_off(dh, 1), &tm_k, p.k_ax, kfull, dh * 64, r1, x.h, x.b);
              }
#pragma unroll
              for (int dh = 0; dh < D / 64; ++dh) {
                load_tile64(vd + pair_off(dh, 0), &tm_v, p.v_ax, vfull, dh * 64, r0, x.h, x.b);
                load_tile64(vd + pair_off(dh, 1), &tm_v, p.v_ax, vfull, dh * 64, r1, x.h, x.b);
              }
            }
          }
          ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        }
      }
      if (ok && lane == 0) {
        // drain: every stage's release (a tcgen05 commit) lands before exit
        for (uint32_t t = (g > (uint32_t)kDqNK ? g - kDqNK : 0u); t < g; ++t)
          if (!mbar_wait(bars + L::kKEmpty + (int)(t % kDqNK), (t / kDqNK) & 1, abort_flag, p.status)) break;
        for (uint32_t t = (g > (uint32_t)kDqNV ? g - kDqNV : 0u); t < g; ++t)
          if (!mbar_wait(bars + L::kVEmpty + (int)(t % kDqNV), (t / kDqNV) & 1, abort_flag, p.status)) break;
        if (n >= 1) mbar_wait(bars + L::kQEmpty, (n - 1) & 1, abort_flag, p.status);
      }
      __syncwarp();
    } else if (warp == 1) {
      // ===================== MMA issue =====================
      // pair g: S^T(g), dP^T(g); then dQ^T += K2(g-1)^T . dS^T(g-1)
      uint32_t g = 0, n = 0;
      bool ok = true;
      for (long long it = it0; ok && it < n_items; it += it_step, ++n) {
        const BwdItem x = load_q_item(p, it);
        const int np = (x.num + 1) / 2, o = (int)(n & 1);
        if (!warp_wait(bars + L::kQFull, n & 1, abort_flag, p.status)) { ok = false; break; }
        const uint32_t g0 = g;
        for (int i = 0; i <= np; ++i) {
          if (i < np) {
            const uint32_t t = g0 + i;
            const int st = (int)(t & 1);
            const int ks = (int)(t % kDqNK), vs = (int)(t % kDqNV);
            if (!warp_wait(bars + L::kKFull + ks, (t / kDqNK) & 1, abort_flag, p.status)) { ok = false; break; }
            if (!warp_wait(bars + L::kVFull + vs, (t / kDqNV) & 1, abort_flag, p.status)) { ok = false; break; }
            if (t >= 2 && !warp_wait(bars + L::kSPEmpty + st, ((t - 2) >> 1) & 1, abort_flag, p.status)) { ok = false; break; }
            if (lane == 0) smeta[st] = meta[ks];
            __syncwarp();
            tc_fence_after_sync();
            if (elect_one()) {
              mma_pair_single<D>(tmem + 64u * st, sbase + L::kKOff + ks * L::kPair, sbase + L::kQOff);
              mma_pair_single<D>(tmem + 128u + 64u * st, sbase + L::kVOff + vs * L::kPair, sbase + L::kDOOff);
              umma_commit(bars + L::kSPFull + st);
              umma_commit(bars + L::kVEmpty + vs);   // V is read by dP only
              if (i == np - 1) umma_commit(bars + L::kQEmpty);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bars + L::kSPFull + st);
          }
          if (i >= 1) {
            const uint32_t t = g0 + i - 1;
            const int st = (int)(t & 1);
            const int ks = (int)(t % kDqNK);
            if (i == 1 && n >= 2 && !warp_wait(bars + L::kOEmpty + o, ((n - 2) >> 1) & 1, abort_flag, p.status)) { ok = false; break; }
            if (!warp_wait(bars + L::kDSFull + st, (t >> 1) & 1, abort_flag, p.status)) { ok = false; break; }
            tc_fence_after_sync();
            if (elect_one()) {
              mma_pairT_mn<D>(tmem + 256u + 64u * o, sbase + L::kKOff + ks * L::kPair,
                              sbase + L::kSOff + st * 16384u, i > 1);
              umma_commit(bars + L::kDSEmpty + st);
              umma_commit(bars + L::kKEmpty + ks);
              if (i == np) umma_commit(bars + L::kOFull + o);
            }
            __syncwarp();
          }
        }
        if (!ok) break;
        if (np == 0) {
          if (n >= 2 && !warp_wait(bars + L::kOEmpty + o, ((n - 2) >> 1) & 1, abort_flag, p.status)) { ok = false; break; }
          if (elect_one()) {
            umma_commit(bars + L::kQEmpty);
            umma_commit(bars + L::kOFull + o);
          }
          __syncwarp();
        }
        g += np;
      }
    }
  } else if (warp < 12) {
    regs_inc<kRegsCompute>();
    // ===================== dS^T = P^T * (dP^T - delta) =====================
    const int grp = (warp - 4) >> 2;        // query columns 32*grp .. 32*grp+31
    const int wq = warp & 3;
    const int Lr = wq * 32 + lane;          // TMEM lane: key row of the pair
    const int half = Lr >> 6, r = Lr & 63;
    const uint32_t col0 = 32u * grp;
    const uint32_t t_lane = tmem + (uint32_t(wq * 32) << 16);
    const float c = p.scale_log2;
    const uint64_t cc = pk2(c, c);
    uint32_t g = 0;
    bool aborted = false;
    auto wwait = [&](uint64_t* bar, uint32_t parity) {
      if (!aborted && !warp_wait(bar, parity, abort_flag, p.status)) aborted = true;
    };
    for (long long it = it0; !aborted && it < n_items; it += it_step) {
      const BwdItem x = load_q_item(p, it);
      const int np = (x.num + 1) / 2;
      // this group's 32 query columns: -lse (log2 units) and delta
      float nl[32], dl[32];
      const long long row0 = x.group * p.q_seq + x.q_tok + col0;
#pragma unroll
      for (int q = 0; q < 32; ++q) {
        const bool real = (int)col0 + q < x.q_len;
        nl[q] = real ? -p.lse[row0 + q] * kLog2e : 0.f;
        dl[q] = real ? p.delta[row0 + q] : 0.f;
      }
      for (int i = 0; i < np; ++i, ++g) {
        const int st = (int)(g & 1);
        wwait(bars + L::kSPFull + st, (g >> 1) & 1);
        const int2 lens = smeta[st];
        const bool valid = r < (half ? lens.y : lens.x);
        tc_fence_after_sync();
        uint32_t sv[32], dv[32];
        VSA_TMEM_LD16(t_lane + 64u * st + col0, sv, 0);
        VSA_TMEM_LD16(t_lane + 64u * st + col0 + 16u, sv, 16);
        VSA_TMEM_LD16(t_lane + 128u + 64u * st + col0, dv, 0);
        VSA_TMEM_LD16(t_lane + 128u + 64u * st + col0 + 16u, dv, 16);
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(bars + L::kSPEmpty + st);
        uint32_t pk[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          float a, b;
          upk2(ffma2(pk2(__uint_as_float(sv[2 * q]), __uint_as_float(sv[2 * q + 1])), cc,
                     pk2(nl[2 * q], nl[2 * q + 1])), a, b);
          float p0 = fast_exp2(a), p1 = fast_exp2(b);
          float d0 = p0 * (__uint_as_float(dv[2 * q]) - dl[2 * q]);
          float d1 = p1 * (__uint_as_float(dv[2 * q + 1]) - dl[2 * q + 1]);
          if (!valid || (int)col0 + 2 * q >= x.q_len) d0 = 0.f;
          if (!valid || (int)col0 + 2 * q + 1 >= x.q_len) d1 = 0.f;
          pk[q] = pack_bf16x2(d0, d1);
        }
        // this dS^T buffer is free once the dQ product of pair g - 2 is done
        if (g >= 2) wwait(bars + L::kDSEmpty + st, ((g - 2) >> 1) & 1);
        uint8_t* sbuf = smem + L::kSOff + st * 16384u;
#pragma unroll
        for (int ch = 0; ch < 4; ++ch)
          *reinterpret_cast<uint4*>(sbuf + sw128(Lr, 4 * grp + ch)) =
              make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bars + L::kDSFull + st);
      }
    }
  } else {
    regs_dec<kRegsEpilogue>();
    // ===================== epilogue: scale * dQ^T -> dq rows =====================
    // thread = head dim d (TMEM lane of dQ^T); rows straight from registers
    const int wq = warp & 3;
    const int d = wq * 32 + lane;
    const uint32_t t_lane = tmem + (uint32_t(wq * 32) << 16);
    const bool active = wq * 32 < D;
    uint32_t n = 0;
    for (long long it = it0; it < n_items; it += it_step, ++n) {
      const BwdItem x = load_q_item(p, it);
      const int o = (int)(n & 1);
      const bool bad = !warp_wait(bars + L::kOFull + o, (n >> 1) & 1, abort_flag, p.status);
      if (bar_red_or(5, 128, bad)) break;
      tc_fence_after_sync();
      __nv_bfloat16* col = p.dq + x.b * p.dq_st.b + x.h * p.dq_st.h + x.q_tok * p.dq_st.s + d;
      for (int rnd = 0; rnd < 4; ++rnd) {
        uint32_t ov[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) ov[q] = 0u;
        if (active && x.num > 0) {
          VSA_TMEM_LD16(t_lane + 256u + 64u * o + 16u * rnd, ov, 0);
          asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
        }
        if (rnd == 3) {
          // the last read of this dQ^T buffer: hand it back before the stores
          tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive(bars + L::kOEmpty + o);
        }
        if (active) {
          float v[16];
#pragma unroll
          for (int q = 0; q < 16; ++q) v[q] = __uint_as_float(ov[q]) * p.scale;
          store_cols_t(col, p.dq_st.s, v, 16 * rnd, x.q_len, p.varlen != 0, lane);
        }
      }
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, 512);
  }
}

// --------------------------------------------------------------------------
// dk / dv kernel
// --------------------------------------------------------------------------
template <int D>
struct DkvLayout {
  static constexpr uint32_t kTile = 64u * D * 2u;
  static constexpr uint32_t kPair = 2u * kTile;
  static constexpr uint32_t kKOff = 0;                   // K tile of the item
  static constexpr uint32_t kVOff = kKOff + kTile;       // V tile
  static constexpr uint32_t kQOff = kVOff + kTile;       // [2] Q pairs (two query blocks)
  static constexpr uint32_t kDOOff = kQOff + 2 * kPair;  // [2] dO pairs
  static constexpr uint32_t kPOff = kDOOff + 2 * kPair;  // [2] P [128][64] bf16
  static constexpr uint32_t kSOff = kPOff + 2u * 16384u; // [2] dS [128][64] bf16
  static constexpr uint32_t kMetaOff = kSOff + 2u * 16384u;  // [2] int4: blocks, multiplicities
  static constexpr uint32_t kSMetaOff = kMetaOff + 32u;      // [2] int4 per TMEM buffer
  static constexpr uint32_t kBarOff = kSMetaOff + 32u;
  static constexpr int kKVFull = 0, kKVEmpty = 1, kQFull = 2, kQEmpty = 4, kSPFull = 6,
                       kSPEmpty = 8, kPSFull = 10, kPSEmpty = 12, kOFull = 14, kOEmpty = 16,
                       kNumBars = 18;
  static constexpr uint32_t kMiscOff = kBarOff + 8u * kNumBars;
  static constexpr uint32_t kAlloc = kMiscOff + 16u + 1024u;
  static_assert(kQOff % 1024 == 0 && kPOff % 1024 == 0, "1 KB atoms");
  static_assert(kAlloc <= 227u * 1024u, "shared memory");
};

struct KvItem {
  int c, h, b;
  long long group;
  int num;          // query blocks listing c
  int kv_len;
  long long kv_tok;
};

__device__ __forceinline__ KvItem load_kv_item(const BwdParams& p, long long it) {
  KvItem x;
  x.c = (int)(it % p.nkv);
  const long long t = it / p.nkv;
  x.h = (int)(t % p.H);
  x.b = (int)(t / p.H);
  x.group = t;
  x.num = p.k2q_num[t * p.nkv + x.c];
  x.kv_tok = p.kv_tok ? (long long)p.kv_tok[x.c] : 64LL * x.c;
  const int l = p.kv_bs ? p.kv_bs[x.c] : 64;
  x.kv_len = (l < 1 || l > 64) ? 0 : l;
  return x;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    dkv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
               const BwdParams p) {
  using L = DkvLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  int4* meta = reinterpret_cast<int4*>(smem + L::kMetaOff);
  int4* smeta = reinterpret_cast<int4*>(smem + L::kSMetaOff);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const long long n_items = (long long)p.B * p.H * p.nkv;
  const long long it0 = blockIdx.x, it_step = gridDim.x;

  if (tid == 0) {
    for (int i = 0; i < L::kNumBars; ++i) {
      uint32_t count = 1;
      if (i == L::kSPEmpty || i == L::kSPEmpty + 1 || i == L::kPSFull || i == L::kPSFull + 1)
        count = 8;
      if (i == L::kOEmpty || i == L::kOEmpty + 1) count = 4;
      if (i == L::kSPFull || i == L::kSPFull + 1) count = 2;
      mbar_init(bars + i, count);
    }
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_do);
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  // TMEM: S at 0, 64; dP at 128, 192; dV^T at 256, 320; dK^T at 384, 448

  if (warp < 4) {
    regs_dec<kRegsProducer>();
    if (warp == 0) {
      // ===================== loads =====================
      uint32_t g = 0, n = 0;
      bool ok = true;
      for (long long it = it0; ok && it < n_items; it += it_step, ++n) {
        const KvItem x = load_kv_item(p, it);
        if (lane == 0) {
          if (n >= 1) ok = mbar_wait(bars + L::kKVEmpty, (n - 1) & 1, abort_flag, p.status);
          if (ok) {
            mbar_arrive_expect_tx(bars + L::kKVFull, 2 * L::kTile);
#pragma unroll
            for (int dh = 0; dh < D / 64; ++dh) {
              load_tile64(smem + L::kKOff + dh * 8192, &tm_k, p.k_ax, bars + L::kKVFull, dh * 64, (int)x.kv_tok, x.h, x.b);
              load_tile64(smem + L::kVOff + dh * 8192, &tm_v, p.v_ax, bars + L::kKVFull, dh * 64, (int)x.kv_tok, x.h, x.b);
            }
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        const int32_t* list = p.k2q + (x.group * p.nkv + x.c) * (long long)p.nq;
        const int np = (x.num + 1) / 2;
        for (int i = 0; ok && i < np; ++i, ++g) {
          if (lane == 0) {
            const int st = (int)(g & 1);
            if (g >= 2) ok = mbar_wait(bars + L::kQEmpty + st, ((g - 2) >> 1) & 1, abort_flag, p.status);
            if (ok) {
              const int e0 = list[2 * i];
              const int e1 = (2 * i + 1 < x.num) ? list[2 * i + 1] : e0;
              const int a0 = e0 & 0xFFFF, a1 = e1 & 0xFFFF;
              const int m0 = e0 >> 16, m1 = (2 * i + 1 < x.num) ? (e1 >> 16) : 0;
              const int t0 = p.q_tok ? p.q_tok[a0] : 64 * a0;
              const int t1 = p.q_tok ? p.q_tok[a1] : 64 * a1;
              const int ql0 = p.q_bs ? p.q_bs[a0] : 64, ql1 = p.q_bs ? p.q_bs[a1] : 64;
              // per query block: first slot; multiplicities (0: no block) and
              // real rows, 16 bits each
              meta[st] = make_int4(t0, t1, m0 | (m1 << 16), ql0 | (ql1 << 16));
              uint64_t* full = bars + L::kQFull + st;
              mbar_arrive_expect_tx(full, 2 * L::kPair);
              uint8_t* qd = smem + L::kQOff + st * L::kPair;
              uint8_t* dd = smem + L::kDOOff + st * L::kPair;
#pragma unroll
              for (int dh = 0; dh < D / 64; ++dh) {
                load_tile64(qd + pair_off(dh, 0), &tm_q, p.q_ax, full, dh * 64, t0, x.h, x.b);
                load_tile64(qd + pair_off(dh, 1), &tm_q, p.q_ax, full, dh * 64, t1, x.h, x.b);
                load_tile64(dd + pair_off(dh, 0), &tm_do, p.do_ax, full, dh * 64, t0, x.h, x.b);
                load_tile64(dd + pair_off(dh, 1), &tm_do, p.do_ax, full, dh * 64, t1, x.h, x.b);
              }
            }
          }
          ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        }
      }
      if (ok && lane == 0) {
        for (uint32_t t = (g > 2u ? g - 2u : 0u); t < g; ++t)
          if (!mbar_wait(bars + L::kQEmpty + (int)(t & 1), (t >> 1) & 1, abort_flag, p.status)) break;
        if (n >= 1) mbar_wait(bars + L::kKVEmpty, (n - 1) & 1, abort_flag, p.status);
      }
      __syncwarp();
    } else if (warp == 1) {
      // ===================== MMA issue =====================
      // step g: S(g), dP(g); then dV^T += dO2(g-1)^T P, dK^T += Q2(g-1)^T dS
      uint32_t g = 0, n = 0;
      bool ok = true;
      for (long long it = it0; ok && it < n_items; it += it_step, ++n) {
        const KvItem x = load_kv_item(p, it);
        const int np = (x.num + 1) / 2, o = (int)(n & 1);
        if (!warp_wait(bars + L::kKVFull, n & 1, abort_flag, p.status)) { ok = false; break; }
        const uint32_t g0 = g;
        for (int i = 0; i <= np; ++i) {
          if (i < np) {
            const uint32_t t = g0 + i;
            const int st = (int)(t & 1);
            if (!warp_wait(bars + L::kQFull + st, (t >> 1) & 1, abort_flag, p.status)) { ok = false; break; }
            if (t >= 2 && !warp_wait(bars + L::kSPEmpty + st, ((t - 2) >> 1) & 1, abort_flag, p.status)) { ok = false; break; }
            if (lane == 0) smeta[st] = meta[st];
            __syncwarp();
            tc_fence_after_sync();
            if (elect_one()) {
              mma_pair_single<D>(tmem + 64u * st, sbase + L::kQOff + st * L::kPair, sbase + L::kKOff);
              mma_pair_single<D>(tmem + 128u + 64u * st, sbase + L::kDOOff + st * L::kPair, sbase + L::kVOff);
              umma_commit(bars + L::kSPFull + st);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bars + L::kSPFull + st);
          }
          if (i >= 1) {
            const uint32_t t = g0 + i - 1;
            const int st = (int)(t & 1);
            if (i == 1 && n >= 2 && !warp_wait(bars + L::kOEmpty + o, ((n - 2) >> 1) & 1, abort_flag, p.status)) { ok = false; break; }
            if (!warp_wait(bars + L::kPSFull + st, (t >> 1) & 1, abort_flag, p.status)) { ok = false; break; }
            tc_fence_after_sync();
            if (elect_one()) {
              mma_pairT_mn<D>(tmem + 256u + 64u * o, sbase + L::kDOOff + st * L::kPair,
                              sbase + L::kPOff + st * 16384u, i > 1);
              mma_pairT_mn<D>(tmem + 384u + 64u * o, sbase + L::kQOff + st * L::kPair,
                              sbase + L::kSOff + st * 16384u, i > 1);
              umma_commit(bars + L::kPSEmpty + st);
              umma_commit(bars + L::kQEmpty + st);
              if (i == np) {
                umma_commit(bars + L::kOFull + o);
                umma_commit(bars + L::kKVEmpty);
              }
            }
            __syncwarp();
          }
        }
        if (!ok) break;
        if (np == 0) {
          if (n >= 2 && !warp_wait(bars + L::kOEmpty + o, ((n - 2) >> 1) & 1, abort_flag, p.status)) { ok = false; break; }
          if (elect_one()) {
            umma_commit(bars + L::kKVEmpty);
            umma_commit(bars + L::kOFull + o);
          }
          __syncwarp();
        }
        g += np;
      }
    }
  } else if (warp < 12) {
    regs_inc<kRegsCompute>();
    // ===================== P and dS, one query row per thread =====================
    const int grp = (warp - 4) >> 2;        // key columns 32*grp .. 32*grp+31
    const int wq = warp & 3;
    const int row = wq * 32 + lane;         // TMEM lane: query row of the pair
    const int half = row >> 6, r = row & 63;
    const uint32_t col0 = 32u * grp;
    const uint32_t t_lane = tmem + (uint32_t(wq * 32) << 16);
    const float c = p.scale_log2;
    const uint64_t cc = pk2(c, c);
    uint32_t g = 0;
    bool aborted = false;
    auto wwait = [&](uint64_t* bar, uint32_t parity) {
      if (!aborted && !warp_wait(bar, parity, abort_flag, p.status)) aborted = true;
    };
    for (long long it = it0; !aborted && it < n_items; it += it_step) {
      const KvItem x = load_kv_item(p, it);
      const int np = (x.num + 1) / 2;
      for (int i = 0; i < np; ++i, ++g) {
        const int st = (int)(g & 1);
        wwait(bars + L::kSPFull + st, (g >> 1) & 1);
        const int4 mt = smeta[st];
        const int mult = half ? ((unsigned)mt.z >> 16) : (mt.z & 0xFFFF);
        const int q_len = half ? ((unsigned)mt.w >> 16) : (mt.w & 0xFFFF);
        const long long tok = (long long)(half ? mt.y : mt.x) + r;
        const bool real = mult > 0 && r < q_len;
        // this row's -lse (log2 units), delta and weight
        const long long ri = x.group * p.q_seq + tok;
        const float nl = real ? -p.lse[ri] * kLog2e : 0.f;
        const float dl = real ? p.delta[ri] : 0.f;
        const float w = real ? (float)mult : 0.f;
        tc_fence_after_sync();
        uint32_t sv[32], dv[32];
        VSA_TMEM_LD16(t_lane + 64u * st + col0, sv, 0);
        VSA_TMEM_LD16(t_lane + 64u * st + col0 + 16u, sv, 16);
        VSA_TMEM_LD16(t_lane + 128u + 64u * st + col0, dv, 0);
        VSA_TMEM_LD16(t_lane + 128u + 64u * st + col0 + 16u, dv, 16);
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(bars + L::kSPEmpty + st);
        uint32_t pp[16], ps[16];
        const uint64_t nl2 = pk2(nl, nl);
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          float a, b;
          upk2(ffma2(pk2(__uint_as_float(sv[2 * q]), __uint_as_float(sv[2 * q + 1])), cc, nl2), a, b);
          float p0 = fast_exp2(a) * w, p1 = fast_exp2(b) * w;
          if ((int)col0 + 2 * q >= x.kv_len || !real) p0 = 0.f;
          if ((int)col0 + 2 * q + 1 >= x.kv_len || !real) p1 = 0.f;
          const float d0 = p0 * (__uint_as_float(dv[2 * q]) - dl);
          const float d1 = p1 * (__uint_as_float(dv[2 * q + 1]) - dl);
          pp[q] = pack_bf16x2(p0, p1);
          ps[q] = pack_bf16x2(d0, d1);
        }
        // this P / dS buffer pair is free once the products of step g - 2 are done
        if (g >= 2) wwait(bars + L::kPSEmpty + st, ((g - 2) >> 1) & 1);
        uint8_t* pbuf = smem + L::kPOff + st * 16384u;
        uint8_t* sbuf = smem + L::kSOff + st * 16384u;
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          *reinterpret_cast<uint4*>(pbuf + sw128(row, 4 * grp + ch)) =
              make_uint4(pp[4 * ch], pp[4 * ch + 1], pp[4 * ch + 2], pp[4 * ch + 3]);
          *reinterpret_cast<uint4*>(sbuf + sw128(row, 4 * grp + ch)) =
              make_uint4(ps[4 * ch], ps[4 * ch + 1], ps[4 * ch + 2], ps[4 * ch + 3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bars + L::kPSFull + st);
      }
    }
  } else {
    regs_dec<kRegsEpilogue>();
    // ===================== epilogue: dV^T, scale * dK^T -> dv, dk rows =====================
    // thread = head dim d (TMEM lane of dV^T / dK^T); rows straight from registers
    const int wq = warp & 3;
    const int d = wq * 32 + lane;
    const uint32_t t_lane = tmem + (uint32_t(wq * 32) << 16);
    const bool active = wq * 32 < D;
    uint32_t n = 0;
    for (long long it = it0; it < n_items; it += it_step, ++n) {
      const KvItem x = load_kv_item(p, it);
      const int o = (int)(n & 1);
      const bool bad = !warp_wait(bars + L::kOFull + o, (n >> 1) & 1, abort_flag, p.status);
      if (bar_red_or(5, 128, bad)) break;
      tc_fence_after_sync();
      for (int which = 0; which < 2; ++which) {
        const Strides3 st = which ? p.dk_st : p.dv_st;
        __nv_bfloat16* col = (which ? p.dk : p.dv) + x.b * st.b + x.h * st.h + x.kv_tok * st.s + d;
        const float mul = which ? p.scale : 1.f;
        for (int rnd = 0; rnd < 4; ++rnd) {
          uint32_t ov[16];
#pragma unroll
          for (int q = 0; q < 16; ++q) ov[q] = 0u;
          if (active && x.num > 0) {
            VSA_TMEM_LD16(t_lane + 256u + 128u * which + 64u * o + 16u * rnd, ov, 0);
            asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
          }
          if (which == 1 && rnd == 3) {
            // the last read of this output buffer pair: hand it back
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(bars + L::kOEmpty + o);
          }
          if (active) {
            float v[16];
#pragma unroll
            for (int q = 0; q < 16; ++q) v[q] = __uint_as_float(ov[q]) * mul;
            store_cols_t(col, st.s, v, 16 * rnd, x.kv_len, p.varlen != 0, lane);
          }
        }
      }
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace bwd

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
static int sm_count_now() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

template <typename Kern>
static int check_regs(Kern kern, int* cache) {
  if (*cache < 0) {
    cudaFuncAttributes attr;
    *cache = (cudaFuncGetAttributes(&attr, kern) == cudaSuccess && attr.numRegs == 128) ? 1 : 0;
  }
  return *cache;
}

template <int D>
static int launch_bwd_t(const BwdParams& p, const CUtensorMap& mq, const CUtensorMap& mk,
                        const CUtensorMap& mv, const CUtensorMap& mdo, cudaStream_t st) {
  static int ok_dq = -1, ok_dkv = -1;
  auto kdq = bwd::dq_kernel<D>;
  auto kdkv = bwd::dkv_kernel<D>;
  if (!check_regs(kdq, &ok_dq) || !check_regs(kdkv, &ok_dkv)) return VSA_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(kdq, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)bwd::DqLayout<D>::kAlloc) != cudaSuccess ||
      cudaFuncSetAttribute(kdkv, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)bwd::DkvLayout<D>::kAlloc) != cudaSuccess)
    return VSA_ERR_CUDA;
  const int sms = sm_count_now();
  const long long nq_items = (long long)p.B * p.H * p.nq, nkv_items = (long long)p.B * p.H * p.nkv;
  kdq<<<(unsigned)(nq_items < sms ? nq_items : sms), bwd::kThreads, bwd::DqLayout<D>::kAlloc, st>>>(
      mq, mk, mv, mdo, p);
  if (cudaGetLastError() != cudaSuccess) return VSA_ERR_CUDA;
  kdkv<<<(unsigned)(nkv_items < sms ? nkv_items : sms), bwd::kThreads, bwd::DkvLayout<D>::kAlloc, st>>>(
      mq, mk, mv, mdo, p);
  return cudaGetLastError() == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

int launch_backward(const BwdParams& p_in, const void* out, Strides3 out_st, int D, cudaStream_t st) {
  if (p_in.B <= 0 || p_in.H <= 0 || p_in.nq <= 0 || p_in.nkv <= 0) return VSA_OK;
  if (p_in.q_seq + 64 > 0x7FFFFFFFLL || p_in.kv_seq + 64 > 0x7FFFFFFFLL) return VSA_ERR_UNSUPPORTED;
  BwdParams p = p_in;
  // delta over every query row
  const long long rows = (long long)p.B * p.H * p.q_seq;
  const long long threads = rows * (D / 8);
  if (D == 128)
    bwd::delta_kernel<128><<<(unsigned)((threads + 255) / 256), 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(out), out_st, p.dout, p.do_st, p.H, p.q_seq, rows, p.delta);
  else
    bwd::delta_kernel<64><<<(unsigned)((threads + 255) / 256), 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(out), out_st, p.dout, p.do_st, p.H, p.q_seq, rows, p.delta);
  if (cudaGetLastError() != cudaSuccess) return VSA_ERR_CUDA;
  // k2q from the selection (index rows staged in shared memory when they fit)
  const size_t k2q_smem = (size_t)p.nq * p.idx_stride * sizeof(int32_t);
  const dim3 kgrid((unsigned)((p.nkv + 7) / 8), (unsigned)(p.B * p.H));
  if (k2q_smem <= 200u * 1024u) {
    if (cudaFuncSetAttribute(bwd::k2q_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)k2q_smem) != cudaSuccess)
      return VSA_ERR_CUDA;
    bwd::k2q_kernel<true><<<kgrid, 256, k2q_smem, st>>>(p.q2k_idx, p.q2k_num, p.nq, p.nkv,
                                                        p.idx_stride, p.q_kv_base, p.q_kv_count,
                                                        p.k2q, p.k2q_num);
  } else {
    bwd::k2q_kernel<false><<<kgrid, 256, 0, st>>>(p.q2k_idx, p.q2k_num, p.nq, p.nkv, p.idx_stride,
                                                  p.q_kv_base, p.q_kv_count, p.k2q, p.k2q_num);
  }
  if (cudaGetLastError() != cudaSuccess) return VSA_ERR_CUDA;
  CUtensorMap mq, mk, mv, mdo;
  if (!make_view_map_rows(&mq, &p.q_ax, p.q, D, p.q_seq, p.H, p.B, p.q_st, 64) ||
      !make_view_map_rows(&mk, &p.k_ax, p.k, D, p.kv_seq, p.H, p.B, p.k_st, 64) ||
      !make_view_map_rows(&mv, &p.v_ax, p.v, D, p.kv_seq, p.H, p.B, p.v_st, 64) ||
      !make_view_map_rows(&mdo, &p.do_ax, p.dout, D, p.q_seq, p.H, p.B, p.do_st, 64))
    return VSA_ERR_CUDA;
  return D == 128 ? launch_bwd_t<128>(p, mq, mk, mv, mdo, st) : launch_bwd_t<64>(p, mq, mk, mv, mdo, st);
}


// ---------------------------------------------------------------------------
// Selection over 128- or 256-slot blocks -> the same selection over 64-slot
// sub-blocks, so the 64-slot backward kernels serve the larger tiles.  One
// warp per (group, query block) index row; the sub-block sizes are written
// by a grid-stride loop over all threads first.
// ---------------------------------------------------------------------------
namespace bwd {

__global__ void __launch_bounds__(256) expand_selection_kernel(ExpandParams e) {
  const int r = 1 << e.shift, blk = 64 << e.shift;
  const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long n_threads = (long long)gridDim.x * blockDim.x;
  const long long n_qsub = (long long)e.nq << e.shift;
  const long long n_sub = n_qsub + ((long long)e.nkv << e.shift);
  for (long long i = tid; i < n_sub; i += n_threads) {
    const bool is_q = i < n_qsub;
    const long long j = is_q ? i : i - n_qsub;
    const int32_t* bs = is_q ? e.q_bs : e.kv_bs;
    int len = bs ? bs[j >> e.shift] : blk;
    len = (len < 1 ? 0 : (len > blk ? blk : len)) - 64 * (int)(j & (r - 1));
    (is_q ? e.q_bs64 : e.kv_bs64)[j] = len < 0 ? 0 : (len > 64 ? 64 : len);
  }
  const long long w = tid >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= e.groups * e.nq) return;
  const int a = (int)(w % e.nq);
  int n = e.q2k_num[w];
  if (n < 0 || n > e.idx_stride) {
    if (lane == 0) set_status(e.status, VSA_ERR_INDEX_RANGE);
    n = n < 0 ? 0 : e.idx_stride;
  }
  int ql = e.q_bs ? e.q_bs[a] : blk;
  ql = ql < 1 ? 0 : (ql > blk ? blk : ql);
  const int32_t* row = e.q2k_idx + w * (long long)e.idx_stride;
  const long long stride64 = (long long)e.idx_stride << e.shift;
  int32_t* out0 = e.idx64 + (w << e.shift) * stride64;  // sub-row i at out0 + i * stride64
  int total = 0;
  for (int j0 = 0; j0 < n; j0 += 32) {
    const int j = j0 + lane;
    int c = 0, cnt = 0;
    if (j < n) {
      c = row[j];
      if (c < 0 || c >= e.nkv) {
        set_status(e.status, VSA_ERR_INDEX_RANGE);
      } else {
        int kl = e.kv_bs ? e.kv_bs[c] : blk;
        kl = kl < 1 ? 0 : (kl > blk ? blk : kl);
        cnt = (kl + 63) >> 6;                    // sub-blocks holding real keys
      }
    }
    int inc = cnt;                               // inclusive prefix over the warp
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += y;
    }
    const int pos = total + inc - cnt;
    for (int s = 0; s < cnt; ++s)
      for (int i = 0; i < r; ++i)
        if (ql > 64 * i) out0[i * stride64 + pos + s] = (c << e.shift) + s;
    total += __shfl_sync(0xffffffffu, inc, 31);
  }
  if (lane < r) e.num64[(w << e.shift) + lane] = ql > 64 * lane ? total : 0;
}

}  // namespace bwd

int launch_expand_selection(const ExpandParams& e, cudaStream_t st) {
  if (e.groups <= 0 || e.nq <= 0 || e.nkv <= 0) return VSA_OK;
  if (e.shift < 1 || e.shift > 2) return VSA_ERR_UNSUPPORTED;
  const long long threads = e.groups * e.nq * 32;
  bwd::expand_selection_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, st>>>(e);
  return cudaGetLastError() == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

}  // namespace vsa
