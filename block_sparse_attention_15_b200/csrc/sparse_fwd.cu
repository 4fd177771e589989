// a4 block-sparse attention over the selected 64x64 tiles, with the a5
// coarse/sparse combine fused into the epilogue.
//
// What it computes ("[chore] release fastvideo-kernel 0.3.0",
// block_sparse_attn_from_indices; "[perf] avoid full-sequence materialization
// in VSA coarse/sparse combine", Problem / Change): for query block a, the
// softmax attention of its real rows over the real keys of the KV blocks
// q2k_idx[a][0 : q2k_num[a]], then out = out_c[a] * gate + out_s with out_c
// held per block and never expanded.
//
// How (sm_100a): one CTA per (query block, head, batch), 6 warps.
//   warp 0      TMA producer: Q once, then the selected K/V tiles two at a
//               time into a 2-stage ring (128-byte swizzle, no multicast).
//   warp 1      TMEM owner and MMA issuer (one thread).
//   warps 2-5   softmax, then the epilogue.
// Each step takes a PAIR of selected KV tiles so that both tensor-core
// products run at M = 128 although a query block has only 64 rows:
//   S^T[128 kv][64 q] = K2[128 kv][D] . Q[64 q][D]^T           (K-major A, B)
//   O^T[D][64 q]     += V2[128 kv][D]^T . P^T[128 kv][64 q]      (MN-major A, B)
// S^T and O^T live in TMEM (fp32).  TMEM lane = KV row for S^T, so the
// softmax thread of lane L owns one key row and all 64 query columns; the
// per-query running max m[q] is kept identical in every softmax thread and
// only refreshed (exact column max across lanes) on the first pair and when
// some logit exceeds it by more than 2^8 -- rare, and then O^T and the row
// sums are rescaled.  Row sums l[q] are accumulated per lane and reduced
// across lanes once at the end.  P^T is written to shared memory in bf16 as
// the B operand of the second product.  S^T is double-buffered in TMEM so the
// tensor core computes S(i+1) and PV(i-1) while the softmax warps work on
// S(i).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "vsa.h"
#include "vsa_device.cuh"
#include "vsa_launch.h"

namespace vsa {

constexpr int kSparseThreads = 192;
constexpr int kMaxSel = VSA_MAX_BLOCKS;
constexpr uint32_t kTmemCols = 256;   // S buffers at 0 and 64, O^T at 128
constexpr uint32_t kTmemO = 128;

template <int D>
struct SparseSmem {
  static constexpr int DH = D / 64;                         // 64-element d halves
  static constexpr uint32_t kQBytes = 64u * D * 2u;         // one 64-row tile
  static constexpr uint32_t kTileBytes = 64u * D * 2u;
  static constexpr uint32_t kKBytes = 2u * kTileBytes;      // two tiles, M = 128
  static constexpr uint32_t kStageBytes = 2u * kKBytes;     // K2 + V2
  static constexpr uint32_t kPBytes = 128u * 64u * 2u;      // P^T, bf16
  static constexpr uint32_t kQOff = 0;
  static constexpr uint32_t kStageOff = kQBytes;
  static constexpr uint32_t kPOff = kStageOff + 2u * kStageBytes;
  static constexpr uint32_t kSelRowOff = kPOff + 2u * kPBytes;
  static constexpr uint32_t kSelLenOff = kSelRowOff + 4u * kMaxSel;
  static constexpr uint32_t kRedOff = kSelLenOff + kMaxSel;     // [4][64] f32
  static constexpr uint32_t kFinOff = kRedOff + 4u * 64u * 4u;  // [64] f32
  static constexpr uint32_t kMOff = kFinOff + 64u * 4u;        // [64] running max (log2 units)
  static constexpr uint32_t kAlphaOff = kMOff + 64u * 4u;       // [64] rescale factors
  static constexpr uint32_t kInvLOff = kAlphaOff + 64u * 4u;    // [64] 1 / row sum
  static constexpr uint32_t kFlagOff = kInvLOff + 64u * 4u;     // [2][4] int
  static constexpr uint32_t kBarOff = kFlagOff + 64u;           // mbarriers
  static constexpr uint32_t kNumBars = 13;
  static constexpr uint32_t kMiscOff = kBarOff + 8u * kNumBars;  // tmem addr, abort
  static constexpr uint32_t kBytes = kMiscOff + 16u;
  static constexpr uint32_t kAlloc = kBytes + 1024u;            // room to align to 1 KB
  static_assert(kQOff % 1024 == 0 && kStageOff % 1024 == 0 && kPOff % 1024 == 0, "align");
  static_assert(2u * kStageBytes >= 64u * D * 4u, "epilogue tile reuses the stage ring");
};

// K2 tile layout: [dh][2 tiles][64 rows][128 B]; V2: [2 tiles][dh][64 rows][128 B].
template <int D>
__device__ __forceinline__ uint32_t k_slot_off(int dh, int tile) {
  return uint32_t(dh) * 16384u + uint32_t(tile) * 8192u;
}
template <int D>
__device__ __forceinline__ uint32_t v_slot_off(int tile, int dh) {
  return uint32_t(tile) * uint32_t(SparseSmem<D>::DH) * 8192u + uint32_t(dh) * 8192u;
}

// S^T[128][64] = K2 . Q^T: M = 128 key rows, N = 64 query rows, K = D.
template <int D>
__device__ __forceinline__ void issue_score_mma(uint32_t tmem_d, uint32_t k_base, uint32_t q_base) {
  constexpr uint32_t idesc = make_idesc_bf16(128, 64, false, false);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const int dh = kk / 4;
    const uint32_t koff = uint32_t(kk % 4) * 32u;
    const uint64_t a = make_sdesc_sw128(k_base + k_slot_off<D>(dh, 0) + koff, 16u, 1024u);
    const uint64_t b = make_sdesc_sw128(q_base + uint32_t(dh) * 8192u + koff, 16u, 1024u);
    umma_bf16(tmem_d, a, b, idesc, kk > 0 ? 1u : 0u);
  }
}

// O^T[128][64] (+)= V2^T . P^T: M = 128 head-dim rows, N = 64 query rows,
// K = 128 key rows.  Both operands MN-major.  The second 64-row atom of A
// (head dims 64..127) sits 8 KB after the first.  For D = 64 that atom is
// other, in-bounds shared memory: TMEM lanes 64..127 then hold values that no
// one reads (row m of the product depends on row m of A only).
template <int D>
__device__ __forceinline__ void issue_pv_mma(uint32_t tmem_o, uint32_t v_base, uint32_t p_base,
                                             bool accumulate) {
  constexpr uint32_t idesc = make_idesc_bf16(128, 64, true, true);
  constexpr uint32_t lbo = 8192u;
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const int tile = kk / 4;
    const uint32_t roff = uint32_t(kk % 4) * 16u * 128u;
    const uint64_t a = make_sdesc_sw128(v_base + v_slot_off<D>(tile, 0) + roff, lbo, 1024u);
    const uint64_t b = make_sdesc_sw128(p_base + uint32_t(kk) * 2048u, 8192u, 1024u);
    umma_bf16(tmem_o, a, b, idesc, (accumulate || kk > 0) ? 1u : 0u);
  }
}

// Byte offset of 16-byte chunk `chunk` of row `row` in a 128-byte-swizzled
// tile whose rows are 128 bytes (atoms of 8 rows, 1 KB aligned).
__device__ __forceinline__ uint32_t sw128_off(uint32_t row, uint32_t chunk) {
  return row * 128u + ((chunk ^ (row & 7u)) << 4);
}

// Reduce 64 per-thread values column-wise across the 128 softmax threads into
// fin[0..63] (shared memory, visible to all 128 threads on return).  Warp
// stage: recursive halving with shuffles, after which lane l holds columns 2l
// and 2l+1; then the four warps combine through shared memory.
template <bool IsMax>
__device__ __forceinline__ float red_op(float a, float b) {
  return IsMax ? fmaxf(a, b) : a + b;
}

template <bool IsMax>
__device__ __forceinline__ void col_reduce64(const float (&v)[64], float* red, float* fin, int wq,
                                             int lane, int t128) {
  float a[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const bool hi = lane & 16;
    const float keep = hi ? v[j + 32] : v[j];
    const float send = hi ? v[j] : v[j + 32];
    a[j] = red_op<IsMax>(keep, __shfl_xor_sync(0xffffffffu, send, 16));
  }
  float b[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const bool hi = lane & 8;
    const float keep = hi ? a[j + 16] : a[j];
    const float send = hi ? a[j] : a[j + 16];
    b[j] = red_op<IsMax>(keep, __shfl_xor_sync(0xffffffffu, send, 8));
  }
  float c[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const bool hi = lane & 4;
    const float keep = hi ? b[j + 8] : b[j];
    const float send = hi ? b[j] : b[j + 8];
    c[j] = red_op<IsMax>(keep, __shfl_xor_sync(0xffffffffu, send, 4));
  }
  float d[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const bool hi = lane & 2;
    const float keep = hi ? c[j + 4] : c[j];
    const float send = hi ? c[j] : c[j + 4];
    d[j] = red_op<IsMax>(keep, __shfl_xor_sync(0xffffffffu, send, 2));
  }
  float e[2];
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const bool hi = lane & 1;
    const float keep = hi ? d[j + 2] : d[j];
    const float send = hi ? d[j] : d[j + 2];
    e[j] = red_op<IsMax>(keep, __shfl_xor_sync(0xffffffffu, send, 1));
  }
  *reinterpret_cast<float2*>(red + wq * 64 + 2 * lane) = make_float2(e[0], e[1]);
  named_barrier_sync(2, 128);
  if (t128 < 64) {
    fin[t128] = red_op<IsMax>(red_op<IsMax>(red[t128], red[64 + t128]),
                              red_op<IsMax>(red[128 + t128], red[192 + t128]));
  }
  named_barrier_sync(2, 128);
}

template <int D, bool COMBINE, bool GATED>
__global__ void __launch_bounds__(kSparseThreads, 1)
    sparse_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const SparseParams p) {
  using L = SparseSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  int32_t* sel_row = reinterpret_cast<int32_t*>(smem + L::kSelRowOff);
  uint8_t* sel_len = smem + L::kSelLenOff;
  float* red = reinterpret_cast<float*>(smem + L::kRedOff);
  float* fin = reinterpret_cast<float*>(smem + L::kFinOff);
  float* m_s = reinterpret_cast<float*>(smem + L::kMOff);
  float* alpha_s = reinterpret_cast<float*>(smem + L::kAlphaOff);
  float* inv_l_s = reinterpret_cast<float*>(smem + L::kInvLOff);
  volatile int* flags = reinterpret_cast<volatile int*>(smem + L::kFlagOff);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* bar_q = bars + 0;
  uint64_t* kv_full = bars + 1;   // [2]
  uint64_t* kv_empty = bars + 3;  // [2]
  uint64_t* s_full = bars + 5;    // [2]
  uint64_t* s_empty = bars + 7;   // [2]
  uint64_t* p_full = bars + 9;    // [2]
  uint64_t* pv_done = bars + 11;  // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);

  const int tid = threadIdx.x;
  const int warp = tid / 32, lane = tid % 32;
  const int a = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const long long group = (long long)b * p.H + h;

  // ---- work item geometry and the selected tiles -------------------------
  int num = p.q2k_num[group * p.nq + a];
  if (num < 0 || num > p.idx_stride) {
    if (tid == 0) set_status(p.status, VSA_ERR_INDEX_RANGE);
    num = num < 0 ? 0 : p.idx_stride;
  }
  const long long q_tok = p.q_tok ? (long long)p.q_tok[a] : 64LL * a;
  int q_len = p.q_bs ? p.q_bs[a] : 64;
  if (q_len < 1 || q_len > 64) {
    if (tid == 0) set_status(p.status, VSA_ERR_BLOCK_SIZE);
    q_len = q_len < 1 ? 0 : 64;
  }
  const int kv_base = p.q_kv_base ? p.q_kv_base[a] : 0;
  const int kv_count = p.q_kv_count ? p.q_kv_count[a] : p.nkv;
  const int32_t* idx_row = p.q2k_idx + (group * p.nq + a) * (long long)p.idx_stride;
  for (int j = tid; j < num; j += kSparseThreads) {
    const int c = idx_row[j];
    int row = 0, len = 0;
    if (c < 0 || c >= kv_count) {
      set_status(p.status, VSA_ERR_INDEX_RANGE);
    } else {
      const int cg = c + kv_base;
      row = p.kv_tok ? p.kv_tok[cg] : 64 * cg;
      len = p.kv_bs ? p.kv_bs[cg] : 64;
      if (len < 1 || len > 64) {
        set_status(p.status, VSA_ERR_BLOCK_SIZE);
        len = 0;
      }
    }
    sel_row[j] = row;
    sel_len[j] = (uint8_t)len;
  }
  if (tid == 0) {
    // s_empty and p_full collect one arrival per softmax warp; the rest one
    // arrival (TMA expect_tx or a tcgen05 commit).
    for (int i = 0; i < (int)L::kNumBars; ++i) {
      const bool per_warp = (bars + i == s_empty) || (bars + i == s_empty + 1) ||
                            (bars + i == p_full) || (bars + i == p_full + 1);
      mbar_init(bars + i, per_warp ? 4u : 1u);
    }
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  const int npairs = (num + 1) / 2;
  const uint32_t q_smem = sbase + L::kQOff;

  if (warp == 0) {
    // ===================== TMA producer =====================
    if (lane == 0 && npairs > 0) {
      const uint64_t pol_q = l2_policy_evict_first();
      const uint64_t pol_kv = l2_policy_evict_last();
      const int q_row = (int)(group * p.q_rows_per_group + q_tok);
      mbar_arrive_expect_tx(bar_q, L::kQBytes);
#pragma unroll
      for (int dh = 0; dh < L::DH; ++dh)
        tma_load_2d(smem + L::kQOff + dh * 8192, &tm_q, bar_q, dh * 64, q_row, pol_q);
      const long long kv_row0 = group * p.kv_rows_per_group;
      for (int i = 0; i < npairs; ++i) {
        const int s = i & 1;
        if (i >= 2 && !mbar_wait(kv_empty + s, ((i - 2) >> 1) & 1, abort_flag, p.status)) break;
        const int j0 = 2 * i;
        const int j1 = (2 * i + 1 < num) ? 2 * i + 1 : 2 * i;
        const int r0 = (int)(kv_row0 + sel_row[j0]);
        const int r1 = (int)(kv_row0 + sel_row[j1]);
        uint8_t* kst = smem + L::kStageOff + s * L::kStageBytes;
        uint8_t* vst = kst + L::kKBytes;
        mbar_arrive_expect_tx(kv_full + s, L::kStageBytes);
#pragma unroll
        for (int dh = 0; dh < L::DH; ++dh) {
          tma_load_2d(kst + k_slot_off<D>(dh, 0), &tm_k, kv_full + s, dh * 64, r0, pol_kv);
          tma_load_2d(kst + k_slot_off<D>(dh, 1), &tm_k, kv_full + s, dh * 64, r1, pol_kv);
        }
#pragma unroll
        for (int dh = 0; dh < L::DH; ++dh) {
          tma_load_2d(vst + v_slot_off<D>(0, dh), &tm_v, kv_full + s, dh * 64, r0, pol_kv);
          tma_load_2d(vst + v_slot_off<D>(1, dh), &tm_v, kv_full + s, dh * 64, r1, pol_kv);
        }
      }
    }
  } else if (warp == 1) {
    // ===================== MMA issuer =====================
    if (lane == 0 && npairs > 0) {
      bool ok = mbar_wait(bar_q, 0, abort_flag, p.status);
      for (int i = 0; ok && i <= npairs; ++i) {
        if (i < npairs) {
          const int s = i & 1;
          if (!mbar_wait(kv_full + s, (i >> 1) & 1, abort_flag, p.status)) break;
          if (i >= 2 && !mbar_wait(s_empty + s, ((i - 2) >> 1) & 1, abort_flag, p.status)) break;
          tc_fence_after_sync();
          issue_score_mma<D>(tmem_base + uint32_t(s) * 64u,
                             sbase + L::kStageOff + s * L::kStageBytes, q_smem);
          umma_commit(s_full + s);
        }
        if (i >= 1) {
          const int j = i - 1, sj = j & 1;
          if (!mbar_wait(p_full + sj, (j >> 1) & 1, abort_flag, p.status)) break;
          tc_fence_after_sync();
          issue_pv_mma<D>(tmem_base + kTmemO,
                          sbase + L::kStageOff + sj * L::kStageBytes + L::kKBytes,
                          sbase + L::kPOff + sj * L::kPBytes, j > 0);
          umma_commit(pv_done + sj);
          // the producer only waits for stages it will refill
          if (j + 2 < npairs) umma_commit(kv_empty + sj);
        }
      }
    }
  } else {
    // ===================== softmax + epilogue (warps 2..5) =====================
    const int wq = warp & 3;             // TMEM lane quarter of this warp
    const int t128 = tid - 64;           // 0..127
    const int Lr = wq * 32 + lane;       // TMEM lane: key row of S^T, d of O^T
    const int half = Lr >> 6, r = Lr & 63;
    const uint32_t t_lane = tmem_base + (uint32_t(wq * 32) << 16);
    const float c = p.scale_log2;
    float lp[64];
#pragma unroll
    for (int q = 0; q < 64; ++q) lp[q] = 0.f;
    bool ok = true;
    for (int i = 0; i < npairs; ++i) {
      const int s = i & 1;
      if (!mbar_wait(s_full + s, (i >> 1) & 1, abort_flag, p.status)) { ok = false; break; }
      tc_fence_after_sync();
      uint32_t sr[64];
      tmem_ld64(t_lane + uint32_t(s) * 64u, sr);
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_empty + s);
      const int jsel = 2 * i + half;
      const int len = (jsel < num) ? (int)sel_len[jsel] : 0;
      const bool valid = r < len;
      bool rescale = (i == 0);
      if (i > 0) {
        // does any logit of this pair exceed the running max by more than 2^8?
        float worst = -INFINITY;
        if (valid) {
#pragma unroll
          for (int q = 0; q < 64; q += 4) {
            const float4 mm = *reinterpret_cast<const float4*>(m_s + q);
            worst = fmaxf(worst, fmaf(__uint_as_float(sr[q]), c, -mm.x));
            worst = fmaxf(worst, fmaf(__uint_as_float(sr[q + 1]), c, -mm.y));
            worst = fmaxf(worst, fmaf(__uint_as_float(sr[q + 2]), c, -mm.z));
            worst = fmaxf(worst, fmaf(__uint_as_float(sr[q + 3]), c, -mm.w));
          }
        }
        const int need = __any_sync(0xffffffffu, worst > 8.f) ? 1 : 0;
        if (lane == 0) flags[(i & 1) * 4 + wq] = need;
        named_barrier_sync(1, 128);
        rescale = (flags[(i & 1) * 4 + 0] | flags[(i & 1) * 4 + 1] | flags[(i & 1) * 4 + 2] |
                   flags[(i & 1) * 4 + 3]) != 0;
      }
      if (rescale) {
        {
          float masked[64];
#pragma unroll
          for (int q = 0; q < 64; ++q) masked[q] = valid ? __uint_as_float(sr[q]) * c : -INFINITY;
          col_reduce64<true>(masked, red, fin, wq, lane, t128);
        }
        if (t128 < 64) {
          const float f = fin[t128];
          if (i == 0) {
            m_s[t128] = (f == -INFINITY) ? 0.f : f;
          } else {
            const float old = m_s[t128];
            const float nm = fmaxf(old, f);
            alpha_s[t128] = fast_exp2(old - nm);
            m_s[t128] = nm;
          }
        }
        named_barrier_sync(2, 128);
        if (i > 0) {
#pragma unroll
          for (int q = 0; q < 64; ++q) lp[q] *= alpha_s[q];
          // O^T already holds PV(0..i-1): wait for the last one, then rescale
          // this thread's lane (one head-dim row, all 64 query columns).
          const int j = i - 1;
          if (!mbar_wait(pv_done + (j & 1), (j >> 1) & 1, abort_flag, p.status)) { ok = false; break; }
          tc_fence_after_sync();
          uint32_t o[64];
          tmem_ld64(t_lane + kTmemO, o);
#pragma unroll
          for (int q = 0; q < 64; ++q) o[q] = __float_as_uint(__uint_as_float(o[q]) * alpha_s[q]);
          tmem_st64(t_lane + kTmemO, o);
          tc_fence_before_sync();
        }
      }
      // probabilities (bf16) for this key row
      uint32_t pk[32];
#pragma unroll
      for (int q = 0; q < 64; q += 4) {
        const float4 mm = *reinterpret_cast<const float4*>(m_s + q);
        float p0 = 0.f, p1 = 0.f, p2 = 0.f, p3 = 0.f;
        if (valid) {
          p0 = fast_exp2(fmaf(__uint_as_float(sr[q]), c, -mm.x));
          p1 = fast_exp2(fmaf(__uint_as_float(sr[q + 1]), c, -mm.y));
          p2 = fast_exp2(fmaf(__uint_as_float(sr[q + 2]), c, -mm.z));
          p3 = fast_exp2(fmaf(__uint_as_float(sr[q + 3]), c, -mm.w));
        }
        lp[q] += p0;
        lp[q + 1] += p1;
        lp[q + 2] += p2;
        lp[q + 3] += p3;
        pk[q / 2] = pack_bf16x2(p0, p1);
        pk[q / 2 + 1] = pack_bf16x2(p2, p3);
      }
      if (i >= 2 && !mbar_wait(pv_done + s, ((i - 2) >> 1) & 1, abort_flag, p.status)) { ok = false; break; }
      uint8_t* pbuf = smem + L::kPOff + s * L::kPBytes;
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {
        *reinterpret_cast<uint4*>(pbuf + sw128_off(Lr, ch)) =
            make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full + s);
    }

    // ---- epilogue --------------------------------------------------------
    float* tile = reinterpret_cast<float*>(smem + L::kStageOff);  // [64][D] fp32
    col_reduce64<false>(lp, red, fin, wq, lane, t128);
    if (t128 < 64) inv_l_s[t128] = fin[t128] > 0.f ? 1.f / fin[t128] : 0.f;
    named_barrier_sync(2, 128);
    bool have_o = ok && npairs > 0;
    if (have_o) {
      const int jl = npairs - 1;
      if (npairs >= 2 && !mbar_wait(pv_done + ((jl - 1) & 1), ((jl - 1) >> 1) & 1, abort_flag, p.status)) have_o = false;
      if (have_o && !mbar_wait(pv_done + (jl & 1), (jl >> 1) & 1, abort_flag, p.status)) have_o = false;
    }
    if (Lr < D) {
      if (have_o) {
        tc_fence_after_sync();
        uint32_t o[64];
        tmem_ld64(t_lane + kTmemO, o);
#pragma unroll
        for (int q = 0; q < 64; ++q) tile[q * D + Lr] = __uint_as_float(o[q]) * inv_l_s[q];
      } else {
#pragma unroll
        for (int q = 0; q < 64; ++q) tile[q * D + Lr] = 0.f;
      }
    } else if (have_o) {
      // D = 64: lanes 64..127 hold nothing of use; the warp still takes
      // part in the collective TMEM load.
      tc_fence_after_sync();
      uint32_t o[64];
      tmem_ld64(t_lane + kTmemO, o);
    }
    tc_fence_before_sync();
    named_barrier_sync(1, 128);
    // cooperative combine + store: 4 consecutive d per thread, coalesced rows
    constexpr int TPR = D / 4;            // threads per row
    constexpr int RPI = 128 / TPR;        // rows per iteration
    const int d0 = (t128 % TPR) * 4;
    const float* oc = COMBINE ? p.out_c + (group * p.nq + a) * (long long)D : nullptr;
    float4 ocv = make_float4(0.f, 0.f, 0.f, 0.f);
    if (COMBINE) ocv = *reinterpret_cast<const float4*>(oc + d0);
    for (int q = t128 / TPR; q < 64; q += RPI) {
      const long long orow = group * p.q_rows_per_group + q_tok + q;
      uint2 packed;
      if (q < q_len) {
        const float4 o = *reinterpret_cast<const float4*>(tile + q * D + d0);
        float v0 = o.x, v1 = o.y, v2 = o.z, v3 = o.w;
        if (COMBINE) {
          if (GATED) {
            const long long grow = ((long long)b * p.gate_seq + q_tok + q) * p.H + h;
            const uint2 graw = *reinterpret_cast<const uint2*>(p.gate + grow * D + d0);
            const float2 g01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&graw.x));
            const float2 g23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&graw.y));
            v0 = fmaf(ocv.x, g01.x, v0);
            v1 = fmaf(ocv.y, g01.y, v1);
            v2 = fmaf(ocv.z, g23.x, v2);
            v3 = fmaf(ocv.w, g23.y, v3);
          } else {
            v0 += ocv.x; v1 += ocv.y; v2 += ocv.z; v3 += ocv.w;
          }
        }
        packed = make_uint2(pack_bf16x2(v0, v1), pack_bf16x2(v2, v3));
      } else {
        if (p.varlen) continue;
        packed = make_uint2(0u, 0u);
      }
      *reinterpret_cast<uint2*>(p.out + orow * D + d0) = packed;
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Self-test of the two products on operands staged by plain loads.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(128, 1)
    selftest_umma_kernel(int mode, const __nv_bfloat16* a, const __nv_bfloat16* bm, float* cm) {
  using L = SparseSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint8_t* opa = smem;                         // 32 KB
  uint8_t* opb = smem + 32768;                 // 16 KB
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + 49152);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + 49152 + 8);
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const uint16_t* a16 = reinterpret_cast<const uint16_t*>(a);
  const uint16_t* b16 = reinterpret_cast<const uint16_t*>(bm);
  if (mode == 0) {
    // a: [128][D] key rows -> K2 layout; b: [64][D] query rows -> Q layout
    for (int e = tid; e < 128 * D; e += 128) {
      const int row = e / D, col = e % D, dh = col / 64, cc = col % 64;
      const int tile = row / 64, rr = row % 64;
      const uint32_t off = k_slot_off<D>(dh, tile) + sw128_off(rr, cc / 8) + (cc % 8) * 2;
      *reinterpret_cast<uint16_t*>(opa + off) = a16[e];
    }
    for (int e = tid; e < 64 * D; e += 128) {
      const int row = e / D, col = e % D, dh = col / 64, cc = col % 64;
      const uint32_t off = dh * 8192 + sw128_off(row, cc / 8) + (cc % 8) * 2;
      *reinterpret_cast<uint16_t*>(opb + off) = b16[e];
    }
  } else {
    // a: [128][D] value rows -> V2 layout; b: [128][64] P^T rows
    for (int e = tid; e < 128 * D; e += 128) {
      const int row = e / D, col = e % D, dh = col / 64, cc = col % 64;
      const int tile = row / 64, rr = row % 64;
      const uint32_t off = v_slot_off<D>(tile, dh) + sw128_off(rr, cc / 8) + (cc % 8) * 2;
      *reinterpret_cast<uint16_t*>(opa + off) = a16[e];
    }
    for (int e = tid; e < 128 * 64; e += 128) {
      const int row = e / 64, col = e % 64;
      const uint32_t off = sw128_off(row, col / 8) + (col % 8) * 2;
      *reinterpret_cast<uint16_t*>(opb + off) = b16[e];
    }
  }
  fence_proxy_async_smem();
  if (tid == 0) {
    mbar_init(bar, 1);
    mbar_fence_init();
  }
  if (warp == 0) tmem_alloc(tmem_slot, 128);
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  if (tid == 0) {
    if (mode == 0) issue_score_mma<D>(tmem_base, sbase, sbase + 32768);
    else issue_pv_mma<D>(tmem_base, sbase, sbase + 32768, false);
    umma_commit(bar);
  }
  int dummy_abort = 0;
  mbar_wait(bar, 0, &dummy_abort, nullptr);
  tc_fence_after_sync();
  uint32_t o[64];
  tmem_ld64(tmem_base + (uint32_t(warp * 32) << 16), o);
  const int row = warp * 32 + lane;
  const int rows = (mode == 0) ? 128 : D;
  if (row < rows) {
    for (int q = 0; q < 64; ++q) cm[row * 64 + q] = __uint_as_float(o[q]);
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, 128);
  }
  (void)L::kBytes;
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult qres;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &qres) ==
            cudaSuccess &&
        qres == cudaDriverEntryPointSuccess) {
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
  }
  return fn;
}

// Row-major [rows][D] bf16 tensor, 64x64 boxes, 128-byte swizzle.
static bool make_tile_map(CUtensorMap* map, const void* base, long long rows, int D) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  cuuint32_t box[2] = {64, 64};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D, bool COMBINE, bool GATED>
static int launch_sparse_t(const SparseParams& p, const CUtensorMap& mq, const CUtensorMap& mk,
                           const CUtensorMap& mv, cudaStream_t stream) {
  using L = SparseSmem<D>;
  auto kern = sparse_fwd_kernel<D, COMBINE, GATED>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::kAlloc) !=
      cudaSuccess)
    return VSA_ERR_CUDA;
  dim3 grid(p.nq, p.H, p.B);
  kern<<<grid, kSparseThreads, L::kAlloc, stream>>>(mq, mk, mv, p);
  return cudaGetLastError() == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

int launch_sparse(const SparseParams& p, const void* q, const void* k, const void* v,
                  long long q_rows_total, long long kv_rows_total, int D, bool combine,
                  bool gated, cudaStream_t stream) {
  if (p.nq <= 0 || p.H <= 0 || p.B <= 0) return VSA_OK;
  if (p.H > 65535 || p.B > 65535) return VSA_ERR_UNSUPPORTED;
  if (q_rows_total + 64 > 0x7FFFFFFFLL || kv_rows_total + 64 > 0x7FFFFFFFLL)
    return VSA_ERR_UNSUPPORTED;  // TMA row coordinates are 32-bit
  CUtensorMap mq, mk, mv;
  if (!make_tile_map(&mq, q, q_rows_total, D) || !make_tile_map(&mk, k, kv_rows_total, D) ||
      !make_tile_map(&mv, v, kv_rows_total, D))
    return VSA_ERR_CUDA;
  if (D == 128) {
    if (!combine) return launch_sparse_t<128, false, false>(p, mq, mk, mv, stream);
    if (gated) return launch_sparse_t<128, true, true>(p, mq, mk, mv, stream);
    return launch_sparse_t<128, true, false>(p, mq, mk, mv, stream);
  }
  if (!combine) return launch_sparse_t<64, false, false>(p, mq, mk, mv, stream);
  if (gated) return launch_sparse_t<64, true, true>(p, mq, mk, mv, stream);
  return launch_sparse_t<64, true, false>(p, mq, mk, mv, stream);
}

int launch_selftest_umma(int mode, int D, const void* a, const void* b, float* c,
                         cudaStream_t stream) {
  const int smem = 49152 + 64 + 1024;
  if (D == 128) {
    cudaFuncSetAttribute(selftest_umma_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    selftest_umma_kernel<128><<<1, 128, smem, stream>>>(
        mode, static_cast<const __nv_bfloat16*>(a), static_cast<const __nv_bfloat16*>(b), c);
  } else {
    cudaFuncSetAttribute(selftest_umma_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    selftest_umma_kernel<64><<<1, 128, smem, stream>>>(
        mode, static_cast<const __nv_bfloat16*>(a), static_cast<const __nv_bfloat16*>(b), c);
  }
  return cudaGetLastError() == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

}  // namespace vsa
