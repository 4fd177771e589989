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
// How (sm_100a).  A query block has 64 rows but tcgen05 runs at full rate
// with M = 128, so every step takes a PAIR of selected KV tiles and both
// products are transposed:
//   S^T[128 kv][64 q] = K2[128 kv][D] . Q[64 q][D]^T           (K-major A, B)
//   O^T[D][64 q]     += V2[128 kv][D]^T . P^T[128 kv][64 q]      (MN-major A, B)
// TMEM lane = key row of S^T (softmax needs no cross-thread work per
// element) and lane = head dim of O^T.  S^T is double-buffered in TMEM and
// O^T too, so the epilogue of one work item overlaps the next item's loop.
//
// Persistent grid: one CTA per SM walks the work items (query block, head,
// batch) b-major, h, a-minor with stride gridDim.x.  512 threads:
//   warp 0       K producer: Q of each item (2 buffers) and K tile pairs into
//                a 3-stage ring, with each pair's key counts (TMA, 128-byte
//                swizzle, no multicast)
//   warp 1       TMEM owner and MMA issuer (one thread)
//   warp 2       V producer: V tile pairs into a 2-stage ring
//   warp 3       idle
//   warps 4-7    softmax for query columns 0..31
//   warps 8-11   softmax for query columns 32..63
//   warps 12-15  epilogue: O^T / l, the gated combine, bf16 stores
// The running max per query column is exact after an item's first pair
// (column reduction across lanes) and refreshed only when a logit exceeds it
// by more than 2^8 (warp vote), then O^T and the partial sums are rescaled.
// Row sums are accumulated per lane and reduced across lanes once per item.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "vsa.h"
#include "vsa_device.cuh"
#include "vsa_launch.h"

namespace vsa {

constexpr int kThreads = 512;
constexpr uint32_t kTmemCols = 256;   // S^T buffers at 0 and 64, O^T buffers at 128 and 192
constexpr uint32_t kTmemO = 128;

template <int D>
struct Layout {
  static constexpr int DH = D / 64;                        // 64-element head-dim halves
  static constexpr int NK = 3;                             // K ring stages (tile pairs)
  static constexpr int NV = 2;                             // V ring stages
  static constexpr uint32_t kQ = 64u * D * 2u;             // one 64-row Q tile
  static constexpr uint32_t kK2 = 2u * 64u * D * 2u;       // a pair of K tiles (M = 128)
  static constexpr uint32_t kV2 = kK2;
  static constexpr uint32_t kP = 128u * 64u * 2u;          // P^T in bf16
  static constexpr uint32_t kQOff = 0;
  static constexpr uint32_t kKOff = kQOff + 2u * kQ;
  static constexpr uint32_t kVOff = kKOff + NK * kK2;
  static constexpr uint32_t kPOff = kVOff + NV * kV2;
  static constexpr uint32_t kRedOff = kPOff + kP;               // [2 groups][4 warps][32] f32
  static constexpr uint32_t kFinOff = kRedOff + 2u * 4u * 32u * 4u;  // [64] f32
  static constexpr uint32_t kMOff = kFinOff + 64u * 4u;         // [64] running max (log2 units)
  static constexpr uint32_t kAlphaOff = kMOff + 64u * 4u;       // [64] rescale factors
  static constexpr uint32_t kInvLOff = kAlphaOff + 64u * 4u;    // [2][64] 1 / row sum per O buffer
  static constexpr uint32_t kFlagOff = kInvLOff + 2u * 64u * 4u;  // [2 groups][2][4] int
  static constexpr uint32_t kKMetaOff = kFlagOff + 64u;         // [NK] int2: key counts of a pair
  static constexpr uint32_t kBarOff = kKMetaOff + 32u;
  // barriers
  static constexpr int kQFull = 0, kQEmpty = 2, kKFull = 4, kKEmpty = kKFull + NK,
                       kVFull = kKEmpty + NK, kVEmpty = kVFull + NV, kSFull = kVEmpty + NV,
                       kSEmpty = kSFull + 2, kPFull = kSEmpty + 2, kPEmpty = kPFull + 1,
                       kOFull = kPEmpty + 1, kOEmpty = kOFull + 2, kLFull = kOEmpty + 2,
                       kNumBars = kLFull + 2;
  static constexpr uint32_t kMiscOff = kBarOff + 8u * kNumBars;  // tmem address, abort flag
  static constexpr uint32_t kBytes = kMiscOff + 16u;
  static constexpr uint32_t kAlloc = kBytes + 1024u;             // slack to align to 1 KB
  static_assert(kKOff % 1024 == 0 && kVOff % 1024 == 0 && kPOff % 1024 == 0, "1 KB atoms");
  static_assert(kAlloc <= 227u * 1024u, "shared memory");
};

// Pair layouts inside a stage.  K2: [dh][2 tiles][64 rows][128 B] (rows of
// the two tiles contiguous, so the pair is one M = 128 operand).
// V2: [2 tiles][dh][64 rows][128 B].
template <int D>
__device__ __forceinline__ uint32_t k_slot_off(int dh, int tile) {
  return uint32_t(dh) * 16384u + uint32_t(tile) * 8192u;
}
template <int D>
__device__ __forceinline__ uint32_t v_slot_off(int tile, int dh) {
  return uint32_t(tile) * uint32_t(D / 64) * 8192u + uint32_t(dh) * 8192u;
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

template <bool IsMax>
__device__ __forceinline__ float red_op(float a, float b) {
  return IsMax ? fmaxf(a, b) : a + b;
}

// Column-wise reduction of 32 per-thread values over the 128 threads of one
// softmax group; the 32 results land in fin[0..31] (shared memory, visible to
// the group on return).  Warp stage: recursive halving with shuffles, after
// which lane l holds column l; then the four warps combine through `red`.
template <bool IsMax>
__device__ __forceinline__ void col_reduce32(const float (&v)[32], float* red, float* fin, int wq,
                                             int lane, int t128, uint32_t bar_id) {
  float a[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const bool hi = lane & 16;
    a[j] = red_op<IsMax>(hi ? v[j + 16] : v[j],
                         __shfl_xor_sync(0xffffffffu, hi ? v[j] : v[j + 16], 16));
  }
  float b[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const bool hi = lane & 8;
    b[j] = red_op<IsMax>(hi ? a[j + 8] : a[j], __shfl_xor_sync(0xffffffffu, hi ? a[j] : a[j + 8], 8));
  }
  float c[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const bool hi = lane & 4;
    c[j] = red_op<IsMax>(hi ? b[j + 4] : b[j], __shfl_xor_sync(0xffffffffu, hi ? b[j] : b[j + 4], 4));
  }
  float d[2];
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const bool hi = lane & 2;
    d[j] = red_op<IsMax>(hi ? c[j + 2] : c[j], __shfl_xor_sync(0xffffffffu, hi ? c[j] : c[j + 2], 2));
  }
  const bool hi = lane & 1;
  const float e = red_op<IsMax>(hi ? d[1] : d[0], __shfl_xor_sync(0xffffffffu, hi ? d[0] : d[1], 1));
  red[wq * 32 + lane] = e;
  named_barrier_sync(bar_id, 128);
  if (t128 < 32) {
    fin[t128] = red_op<IsMax>(red_op<IsMax>(red[t128], red[32 + t128]),
                              red_op<IsMax>(red[64 + t128], red[96 + t128]));
  }
  named_barrier_sync(bar_id, 128);
}

// One work item: query block a of head h of batch b.
struct Item {
  int a, h, b;
  long long group;     // b * H + h
  int num;             // selected entries, clamped to [0, idx_stride]
  int q_len;           // real query rows
  long long q_tok;     // first token row of the block within its group
  int kv_base, kv_count;
};

__device__ __forceinline__ Item load_item(const SparseParams& p, long long it) {
  Item x;
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

// Report a work item whose count or query block size is out of range.
__device__ __forceinline__ void check_item(const SparseParams& p, long long it) {
  const long long t = it / p.nq;
  const int a = (int)(it % p.nq);
  const int num = p.q2k_num[t * p.nq + a];
  if (num < 0 || num > p.idx_stride) set_status(p.status, VSA_ERR_INDEX_RANGE);
  const int ql = p.q_bs ? p.q_bs[a] : 64;
  if (ql < 1 || ql > 64) set_status(p.status, VSA_ERR_BLOCK_SIZE);
}

// Producer helper: for entry j of an item's selection, the row of its first
// token within the group and its key count (0 for an invalid entry, which is
// reported and then masked out).
__device__ __forceinline__ void resolve_entry(const SparseParams& p, const Item& x,
                                              const int32_t* idx_row, int j, int& row, int& len) {
  row = 0;
  len = 0;
  if (j >= x.num) return;
  const int c = idx_row[j];
  if (c < 0 || c >= x.kv_count) {
    set_status(p.status, VSA_ERR_INDEX_RANGE);
    return;
  }
  const int cg = c + x.kv_base;
  row = p.kv_tok ? p.kv_tok[cg] : 64 * cg;
  len = p.kv_bs ? p.kv_bs[cg] : 64;
  if (len < 1 || len > 64) {
    set_status(p.status, VSA_ERR_BLOCK_SIZE);
    len = 0;
  }
}

template <int D, bool COMBINE, bool GATED>
__global__ void __launch_bounds__(kThreads, 1)
    sparse_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const SparseParams p) {
  using L = Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  float* red_all = reinterpret_cast<float*>(smem + L::kRedOff);
  float* fin_all = reinterpret_cast<float*>(smem + L::kFinOff);
  float* m_s = reinterpret_cast<float*>(smem + L::kMOff);
  float* alpha_s = reinterpret_cast<float*>(smem + L::kAlphaOff);
  float* inv_l = reinterpret_cast<float*>(smem + L::kInvLOff);
  volatile int* flags = reinterpret_cast<volatile int*>(smem + L::kFlagOff);
  int2* kmeta = reinterpret_cast<int2*>(smem + L::kKMetaOff);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);

  const int tid = threadIdx.x;
  const int warp = tid / 32, lane = tid % 32;
  const long long n_items = (long long)p.B * p.H * p.nq;
  const long long it0 = blockIdx.x, it_step = gridDim.x;

  if (tid == 0) {
    for (int i = 0; i < L::kNumBars; ++i) {
      uint32_t count = 1;
      if (i == L::kSEmpty || i == L::kSEmpty + 1 || i == L::kPFull || i == L::kLFull ||
          i == L::kLFull + 1)
        count = 8;  // one arrival per softmax warp
      if (i >= L::kKEmpty && i < L::kKEmpty + L::NK) count = 9;  // MMA commit + 8 softmax warps
      if (i == L::kOEmpty || i == L::kOEmpty + 1) count = 4;   // epilogue warps
      mbar_init(bars + i, count);
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

  if (warp == 0 || warp == 2) {
    // ===================== producers (whole warp) =====================
    const bool is_k = (warp == 0);
    const uint64_t pol_q = l2_policy_evict_first();
    const uint64_t pol_kv = l2_policy_evict_last();
    long long gp = 0;  // pair counter over this CTA's items
    bool ok = true;
    long long n = 0;
    for (long long it = it0; ok && it < n_items; it += it_step, ++n) {
      const Item x = load_item(p, it);
      const int o = (int)(n & 1);
      if (is_k) {
        if (lane == 0) {
          check_item(p, it);
          if (n >= 2)
            ok = mbar_wait(bars + L::kQEmpty + o, (uint32_t)(((n - 2) >> 1) & 1), abort_flag, p.status);
          if (ok) {
            mbar_arrive_expect_tx(bars + L::kQFull + o, L::kQ);
            const int q_row = (int)(x.group * p.q_rows_per_group + x.q_tok);
#pragma unroll
            for (int dh = 0; dh < L::DH; ++dh)
              tma_load_2d(smem + L::kQOff + o * L::kQ + dh * 8192, &tm_q, bars + L::kQFull + o,
                          dh * 64, q_row, pol_q);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      }
      const int32_t* idx_row = p.q2k_idx + (x.group * p.nq + x.a) * (long long)p.idx_stride;
      const int np = (x.num + 1) / 2;
      const long long kv_row0 = x.group * p.kv_rows_per_group;
      for (int j0 = 0; ok && j0 < x.num; j0 += 32) {
        int row, len;
        resolve_entry(p, x, idx_row, j0 + lane, row, len);
        const int i_end = min(np, (j0 + 32) / 2);
        for (int i = j0 / 2; i < i_end; ++i) {
          const int r0 = __shfl_sync(0xffffffffu, row, 2 * i - j0);
          const int l0 = __shfl_sync(0xffffffffu, len, 2 * i - j0);
          int r1 = __shfl_sync(0xffffffffu, row, 2 * i + 1 - j0);
          int l1 = __shfl_sync(0xffffffffu, len, 2 * i + 1 - j0);
          if (2 * i + 1 >= x.num) { r1 = r0; l1 = 0; }
          if (lane == 0) {
            if (is_k) {
              const int ks = (int)(gp % L::NK);
              const long long u = gp / L::NK;
              if (u >= 1) ok = mbar_wait(bars + L::kKEmpty + ks, (uint32_t)((u - 1) & 1), abort_flag, p.status);
              if (ok) {
                kmeta[ks] = make_int2(l0, l1);
                uint8_t* dst = smem + L::kKOff + ks * L::kK2;
                mbar_arrive_expect_tx(bars + L::kKFull + ks, L::kK2);
#pragma unroll
                for (int dh = 0; dh < L::DH; ++dh) {
                  tma_load_2d(dst + k_slot_off<D>(dh, 0), &tm_k, bars + L::kKFull + ks, dh * 64,
                              (int)(kv_row0 + r0), pol_kv);
                  tma_load_2d(dst + k_slot_off<D>(dh, 1), &tm_k, bars + L::kKFull + ks, dh * 64,
                              (int)(kv_row0 + r1), pol_kv);
                }
              }
            } else {
              const int vs = (int)(gp % L::NV);
              const long long u = gp / L::NV;
              if (u >= 1) ok = mbar_wait(bars + L::kVEmpty + vs, (uint32_t)((u - 1) & 1), abort_flag, p.status);
              if (ok) {
                uint8_t* dst = smem + L::kVOff + vs * L::kV2;
                mbar_arrive_expect_tx(bars + L::kVFull + vs, L::kV2);
#pragma unroll
                for (int dh = 0; dh < L::DH; ++dh) {
                  tma_load_2d(dst + v_slot_off<D>(0, dh), &tm_v, bars + L::kVFull + vs, dh * 64,
                              (int)(kv_row0 + r0), pol_kv);
                  tma_load_2d(dst + v_slot_off<D>(1, dh), &tm_v, bars + L::kVFull + vs, dh * 64,
                              (int)(kv_row0 + r1), pol_kv);
                }
              }
            }
          }
          ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
          if (!ok) break;
          ++gp;
        }
      }
    }
  } else if (warp == 1) {
    // ===================== MMA issuer =====================
    if (lane == 0) {
      // total pairs and items of this CTA: commits that nobody would wait for
      // are not issued, so no asynchronous arrival outlives the CTA
      long long total = 0, n_mine = 0;
      for (long long it = it0; it < n_items; it += it_step, ++n_mine) {
        const Item x = load_item(p, it);
        total += (x.num + 1) / 2;
      }
      long long gp = 0, n = 0;
      bool ok = true;
      // the PV product runs one step behind the score product
      long long pv_g = -1, pv_n = 0;
      int pv_o = 0;
      bool pv_first = false, pv_last = false;
      auto issue_pv = [&]() -> bool {
        const int vs = (int)(pv_g % L::NV);
        if (!mbar_wait(bars + L::kVFull + vs, (uint32_t)((pv_g / L::NV) & 1), abort_flag, p.status)) return false;
        if (!mbar_wait(bars + L::kPFull, (uint32_t)(pv_g & 1), abort_flag, p.status)) return false;
        if (pv_first && pv_n >= 2 &&
            !mbar_wait(bars + L::kOEmpty + pv_o, (uint32_t)(((pv_n - 2) >> 1) & 1), abort_flag, p.status))
          return false;
        tc_fence_after_sync();
        issue_pv_mma<D>(tmem_base + kTmemO + 64u * pv_o, sbase + L::kVOff + vs * L::kV2,
                        sbase + L::kPOff, !pv_first);
        if (pv_g + 1 < total) umma_commit(bars + L::kPEmpty);
        if (pv_g + L::NV < total) umma_commit(bars + L::kVEmpty + vs);
        if (pv_last) umma_commit(bars + L::kOFull + pv_o);
        pv_g = -1;
        return true;
      };
      for (long long it = it0; ok && it < n_items; it += it_step, ++n) {
        const Item x = load_item(p, it);
        const int o = (int)(n & 1);
        const int np = (x.num + 1) / 2;
        if (!mbar_wait(bars + L::kQFull + o, (uint32_t)((n >> 1) & 1), abort_flag, p.status)) { ok = false; break; }
        for (int i = 0; i < np; ++i, ++gp) {
          const int sb = (int)(gp & 1);
          const int ks = (int)(gp % L::NK);
          if (!mbar_wait(bars + L::kKFull + ks, (uint32_t)((gp / L::NK) & 1), abort_flag, p.status)) { ok = false; break; }
          if (gp >= 2 && !mbar_wait(bars + L::kSEmpty + sb, (uint32_t)(((gp - 2) >> 1) & 1), abort_flag, p.status)) { ok = false; break; }
          tc_fence_after_sync();
          issue_score_mma<D>(tmem_base + 64u * sb, sbase + L::kKOff + ks * L::kK2,
                             sbase + L::kQOff + o * L::kQ);
          umma_commit(bars + L::kSFull + sb);
          if (gp + L::NK < total) umma_commit(bars + L::kKEmpty + ks);
          if (i == np - 1 && n + 2 < n_mine) umma_commit(bars + L::kQEmpty + o);
          if (pv_g >= 0 && !issue_pv()) { ok = false; break; }
          pv_g = gp; pv_n = n; pv_o = o; pv_first = (i == 0); pv_last = (i == np - 1);
        }
        if (!ok) break;
        if (np == 0) {
          // empty selection: no products; still hand the O buffer to the
          // epilogue in order (it writes out_c * gate for this block)
          if (pv_g >= 0 && !issue_pv()) { ok = false; break; }
          if (n >= 2 && !mbar_wait(bars + L::kOEmpty + o, (uint32_t)(((n - 2) >> 1) & 1), abort_flag, p.status)) { ok = false; break; }
          umma_commit(bars + L::kOFull + o);
          if (n + 2 < n_mine) umma_commit(bars + L::kQEmpty + o);
        }
      }
      if (ok && pv_g >= 0) issue_pv();
    }
  } else if (warp >= 4 && warp < 12) {
    // ===================== softmax (two groups of 4 warps) =====================
    const int grp = (warp - 4) / 4;              // query columns 32*grp .. 32*grp+31
    const int wq = warp & 3;                     // TMEM lane quarter
    const int t128 = (warp - 4 - 4 * grp) * 32 + lane;
    const int Lr = wq * 32 + lane;               // TMEM lane: key row of S^T, head dim of O^T
    const int half = Lr >> 6, r = Lr & 63;
    const uint32_t col0 = 32u * grp;
    const uint32_t t_lane = tmem_base + (uint32_t(wq * 32) << 16);
    const uint32_t bar_flag = 1 + 2 * grp, bar_red = 2 + 2 * grp;
    float* red = red_all + grp * 128;
    float* fin = fin_all + col0;
    volatile int* gflags = flags + grp * 8;
    float* m_g = m_s + col0;
    float* a_g = alpha_s + col0;
    const float c = p.scale_log2;
    long long gp = 0, n = 0;
    bool ok = true;
    for (long long it = it0; ok && it < n_items; it += it_step, ++n) {
      const Item x = load_item(p, it);
      const int o = (int)(n & 1);
      const int np = (x.num + 1) / 2;
      float lp[32];
#pragma unroll
      for (int q = 0; q < 32; ++q) lp[q] = 0.f;
      for (int i = 0; i < np; ++i, ++gp) {
        const int sb = (int)(gp & 1);
        const int ks = (int)(gp % L::NK);
        if (!mbar_wait(bars + L::kSFull + sb, (uint32_t)((gp >> 1) & 1), abort_flag, p.status)) { ok = false; break; }
        // the K stage's barrier also publishes the pair's key counts; the
        // stage cannot be refilled before this group's arrival below
        if (!mbar_wait(bars + L::kKFull + ks, (uint32_t)((gp / L::NK) & 1), abort_flag, p.status)) { ok = false; break; }
        const int2 lens = kmeta[ks];
        const bool valid = r < (half ? lens.y : lens.x);
        __syncwarp();
        if (lane == 0) mbar_arrive(bars + L::kKEmpty + ks);
        tc_fence_after_sync();
        uint32_t sr[32];
        tmem_ld32(t_lane + 64u * sb + col0, sr);
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(bars + L::kSEmpty + sb);
        bool rescale = (i == 0);
        if (i > 0) {
          float worst = -INFINITY;
          if (valid) {
#pragma unroll
            for (int q = 0; q < 32; q += 4) {
              const float4 mm = *reinterpret_cast<const float4*>(m_g + q);
              worst = fmaxf(worst, fmaf(__uint_as_float(sr[q]), c, -mm.x));
              worst = fmaxf(worst, fmaf(__uint_as_float(sr[q + 1]), c, -mm.y));
              worst = fmaxf(worst, fmaf(__uint_as_float(sr[q + 2]), c, -mm.z));
              worst = fmaxf(worst, fmaf(__uint_as_float(sr[q + 3]), c, -mm.w));
            }
          }
          const int need = __any_sync(0xffffffffu, worst > 8.f) ? 1 : 0;
          if (lane == 0) gflags[(gp & 1) * 4 + wq] = need;
          named_barrier_sync(bar_flag, 128);
          rescale = (gflags[(gp & 1) * 4 + 0] | gflags[(gp & 1) * 4 + 1] |
                     gflags[(gp & 1) * 4 + 2] | gflags[(gp & 1) * 4 + 3]) != 0;
        }
        if (rescale) {
          {
            float masked[32];
#pragma unroll
            for (int q = 0; q < 32; ++q) masked[q] = valid ? __uint_as_float(sr[q]) * c : -INFINITY;
            col_reduce32<true>(masked, red, fin, wq, lane, t128, bar_red);
          }
          if (t128 < 32) {
            const float f = fin[t128];
            if (i == 0) {
              m_g[t128] = (f == -INFINITY) ? 0.f : f;
            } else {
              const float old = m_g[t128];
              const float nm = fmaxf(old, f);
              a_g[t128] = fast_exp2(old - nm);
              m_g[t128] = nm;
            }
          }
          named_barrier_sync(bar_red, 128);
          if (i > 0) {
#pragma unroll
            for (int q = 0; q < 32; ++q) lp[q] *= a_g[q];
            // O^T holds this item's PV products up to the previous pair:
            // wait for the last one, then rescale this lane's columns.
            if (!mbar_wait(bars + L::kPEmpty, (uint32_t)((gp - 1) & 1), abort_flag, p.status)) { ok = false; break; }
            tc_fence_after_sync();
            uint32_t ov[32];
            tmem_ld32(t_lane + kTmemO + 64u * o + col0, ov);
#pragma unroll
            for (int q = 0; q < 32; ++q) ov[q] = __float_as_uint(__uint_as_float(ov[q]) * a_g[q]);
            tmem_st32(t_lane + kTmemO + 64u * o + col0, ov);
            tc_fence_before_sync();
          }
        }
        uint32_t pk[16];
#pragma unroll
        for (int q = 0; q < 32; q += 4) {
          const float4 mm = *reinterpret_cast<const float4*>(m_g + q);
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
        // the single P^T buffer is free once the previous PV product is done
        if (gp >= 1 && !mbar_wait(bars + L::kPEmpty, (uint32_t)((gp - 1) & 1), abort_flag, p.status)) { ok = false; break; }
        uint8_t* pbuf = smem + L::kPOff;
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          *reinterpret_cast<uint4*>(pbuf + sw128_off(Lr, 4 * grp + ch)) =
              make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bars + L::kPFull);
      }
      if (!ok) break;
      // end of item: 1 / row sums for the epilogue
      if (n >= 2 && !mbar_wait(bars + L::kOEmpty + o, (uint32_t)(((n - 2) >> 1) & 1), abort_flag, p.status)) { ok = false; break; }
      col_reduce32<false>(lp, red, fin, wq, lane, t128, bar_red);
      if (t128 < 32) inv_l[o * 64 + col0 + t128] = fin[t128] > 0.f ? 1.f / fin[t128] : 0.f;
      named_barrier_sync(bar_red, 128);
      __syncwarp();
      if (lane == 0) mbar_arrive(bars + L::kLFull + o);
    }
  } else if (warp >= 12) {
    // ===================== epilogue =====================
    const int wq = warp & 3;
    const int d = wq * 32 + lane;                // TMEM lane = head dim of O^T
    const uint32_t t_lane = tmem_base + (uint32_t(wq * 32) << 16);
    long long n = 0;
    for (long long it = it0; it < n_items; it += it_step, ++n) {
      const Item x = load_item(p, it);
      const int o = (int)(n & 1);
      if (!mbar_wait(bars + L::kOFull + o, (uint32_t)((n >> 1) & 1), abort_flag, p.status)) break;
      if (!mbar_wait(bars + L::kLFull + o, (uint32_t)((n >> 1) & 1), abort_flag, p.status)) break;
      float ov[64];
      if (wq * 32 < D && x.num > 0) {
        tc_fence_after_sync();
        uint32_t raw[32];
        tmem_ld32(t_lane + kTmemO + 64u * o, raw);
#pragma unroll
        for (int q = 0; q < 32; ++q) ov[q] = __uint_as_float(raw[q]) * inv_l[o * 64 + q];
        tmem_ld32(t_lane + kTmemO + 64u * o + 32u, raw);
#pragma unroll
        for (int q = 0; q < 32; ++q) ov[32 + q] = __uint_as_float(raw[q]) * inv_l[o * 64 + 32 + q];
      } else {
#pragma unroll
        for (int q = 0; q < 64; ++q) ov[q] = 0.f;
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(bars + L::kOEmpty + o);
      if (wq * 32 >= D) continue;
      float oc = 0.f;
      if (COMBINE) oc = p.out_c[(x.group * p.nq + x.a) * (long long)D + d];
      const long long orow0 = x.group * p.q_rows_per_group + x.q_tok;
      const long long grow0 = ((long long)x.b * p.gate_seq + x.q_tok) * p.H + x.h;
#pragma unroll
      for (int q = 0; q < 64; ++q) {
        __nv_bfloat16 val;
        if (q < x.q_len) {
          float v = ov[q];
          if (COMBINE) {
            if (GATED) {
              const float g = __bfloat162float(p.gate[(grow0 + (long long)q * p.H) * D + d]);
              v = fmaf(oc, g, v);
            } else {
              v += oc;
            }
          }
          val = __float2bfloat16_rn(v);
        } else {
          if (p.varlen) continue;
          val = __float2bfloat16_rn(0.f);
        }
        p.out[(orow0 + q) * D + d] = val;
      }
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

static int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!cached[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

template <int D, bool COMBINE, bool GATED>
static int launch_sparse_t(const SparseParams& p, const CUtensorMap& mq, const CUtensorMap& mk,
                           const CUtensorMap& mv, cudaStream_t stream) {
  using L = Layout<D>;
  auto kern = sparse_fwd_kernel<D, COMBINE, GATED>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::kAlloc) !=
      cudaSuccess)
    return VSA_ERR_CUDA;
  const long long n_items = (long long)p.B * p.H * p.nq;
  const long long grid = n_items < sm_count() ? n_items : sm_count();
  kern<<<(unsigned)grid, kThreads, L::kAlloc, stream>>>(mq, mk, mv, p);
  return cudaGetLastError() == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

int launch_sparse(const SparseParams& p, const void* q, const void* k, const void* v,
                  long long q_rows_total, long long kv_rows_total, int D, bool combine,
                  bool gated, cudaStream_t stream) {
  if (p.nq <= 0 || p.H <= 0 || p.B <= 0) return VSA_OK;
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
