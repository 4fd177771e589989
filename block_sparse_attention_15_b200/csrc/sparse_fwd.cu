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
// element) and lane = head dim of O^T.  S^T has four TMEM buffers and O^T
// two, so the epilogue of one work item overlaps the next item's loop.
//
// Persistent grid: one CTA per SM walks the work items (query block, head,
// batch) b-major, h, a-minor with stride gridDim.x.  512 threads, four
// warpgroups:
//   warp 0       K producer: the item's Q tile and K tile pairs into a
//                2-stage ring with each pair's key counts (TMA, 128-byte
//                swizzle, no multicast)
//   warp 1       TMEM owner; issues the score products S^T into four TMEM
//                buffers, running ahead of the softmax
//   warp 2       V producer: V tile pairs into a 2-stage ring
//   warp 3       issues the PV products into two TMEM output buffers
//   warps 4-7    softmax for query columns 0..31
//   warps 8-11   softmax for query columns 32..63
//   warps 12-15  epilogue: O^T / l, the gated combine, bf16 stores
// The softmax takes two pairs per step; P^T has shared-memory buffers for
// two steps, so a step waits for the PV products of the step before the
// previous one (and the previous step's run while it computes).  A
// Cauchy-Schwarz bound on an item's logits (largest query row norm of the
// block x largest key row norm of its selected blocks x scale), where it is
// at most kNoClampBound, is every column's reference max from the first
// step on: no step then needs a maximum, a vote or a rescale.  Otherwise the
// running max per query column is exact after an item's first step (column
// reduction across lanes) and refreshed only when a logit exceeds it by more
// than kOffsetLimit (log2 units; barrier vote), then O^T and the partial sums
// are rescaled.  Row sums are accumulated per lane and reduced across lanes
// once per item.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "vsa.h"
#include "vsa_device.cuh"
#include "vsa_launch.h"

namespace vsa {

template <bool B>
struct BoolTag {
  static constexpr bool value = B;
};

constexpr int kThreads = 512;
// registers per thread of the producer / MMA, softmax and epilogue warpgroups
#ifndef VSA_REGS_P
#define VSA_REGS_P 64
#endif
#ifndef VSA_REGS_S
#define VSA_REGS_S 192
#endif
#ifndef VSA_REGS_E
#define VSA_REGS_E 64
#endif
constexpr uint32_t kRegsProducer = VSA_REGS_P, kRegsSoftmax = VSA_REGS_S, kRegsEpilogue = VSA_REGS_E;
static_assert(128u * (kRegsProducer + 2u * kRegsSoftmax + kRegsEpilogue) <= 512u * 128u,
              "register split exceeds the launch's 128 registers per thread");
#ifndef VSA_KLEAD
#define VSA_KLEAD 6
#endif
constexpr int kKLead = VSA_KLEAD;      // K requests run at most this many pairs ahead of V
#ifndef VSA_NS
#define VSA_NS 4
#endif
constexpr int kNS = VSA_NS;            // S^T buffers in TMEM (64 columns each)
#ifndef VSA_NP
#define VSA_NP 4
#endif
#ifndef VSA_POLY8
#define VSA_POLY8 2   // column pairs in eight whose exponential runs on the FMA pipe
#endif
constexpr int kNP = VSA_NP;            // P^T buffers in shared memory (even)
static_assert(kNP >= 2 && kNP % 2 == 0, "two pairs per softmax step");
constexpr uint32_t kTmemCols = 512;    // S^T buffers at 64*i (i < kNS), then the two O^T buffers
constexpr uint32_t kTmemO = 64u * kNS;
static_assert(kTmemO + 128u <= kTmemCols, "S^T and O^T buffers exceed TMEM");
// Largest offset (log2 units) of a logit above its column's running max that
// is exponentiated without a refresh: probabilities stay below 2^32, far from
// fp32 / bf16 overflow in P^T, O^T and the row sums.
constexpr float kOffsetLimit = 32.f;
// Largest logit bound (log2 units) for which an item's vote-free steps skip
// the exponential's lower clamp: every offset s*c - m is then >= -2 * bound
// (s*c >= -bound and the running max m <= bound), so >= -120.
constexpr float kNoClampBound = 60.f;

template <int D>
struct Layout {
  static constexpr int DH = D / 64;                        // 64-element head-dim halves
#ifndef VSA_NK
#define VSA_NK 2
#endif
#ifndef VSA_NV
#define VSA_NV 2
#endif
  static constexpr int NK = VSA_NK;                        // K ring stages (tile pairs)
  static constexpr int NV = VSA_NV;                        // V ring stages
  static constexpr uint32_t kQ = 64u * D * 2u;             // one 64-row Q tile
  static constexpr uint32_t kK2 = 2u * 64u * D * 2u;       // a pair of K tiles (M = 128)
  static constexpr uint32_t kV2 = kK2;
  static constexpr uint32_t kP = 128u * 64u * 2u;          // P^T in bf16
  static constexpr uint32_t kQOff = 0;
  static constexpr uint32_t kKOff = kQOff + kQ;
  static constexpr uint32_t kVOff = kKOff + NK * kK2;
  static constexpr uint32_t kPOff = kVOff + NV * kV2;
  static constexpr uint32_t kStageOff = kPOff + kNP * kP;       // epilogue tile [16][D] f32
  static constexpr uint32_t kRedOff = kStageOff + 16u * D * 4u; // [2 groups][4 warps][32] f32
  static constexpr uint32_t kFinOff = kRedOff + 2u * 4u * 32u * 4u;  // [64] f32
  static constexpr uint32_t kAlphaOff = kFinOff + 64u * 4u;     // [64] rescale factors
  static constexpr uint32_t kMnOff = kAlphaOff + 64u * 4u;      // [64] minus the running max per column
  static constexpr uint32_t kInvLOff = kMnOff + 64u * 4u;       // [2][64] 1 / row sum per O buffer
  static constexpr uint32_t kLseOff = kInvLOff + 2u * 64u * 4u;   // [2][64] log-sum-exp (log2 units)
  static constexpr uint32_t kKMetaOff = kLseOff + 2u * 64u * 4u;  // [NK] int2: key counts
  static constexpr uint32_t kSMetaOff = kKMetaOff + 8u * NK;       // [kNS] int2: key counts per S^T buffer
  static constexpr uint32_t kVIssuedOff = kSMetaOff + 8u * kNS;   // V pairs requested so far
  static constexpr uint32_t kBarOff = kVIssuedOff + 16u;
  // barriers
  static constexpr int kQFull = 0, kQEmpty = 1, kKFull = 2, kKEmpty = kKFull + NK,
                       kVFull = kKEmpty + NK, kVEmpty = kVFull + NV, kSFull = kVEmpty + NV,
                       kSEmpty = kSFull + kNS, kPFull = kSEmpty + kNS, kPEmpty = kPFull + kNP,
                       kOFull = kPEmpty + kNP, kOEmpty = kOFull + 2, kLFull = kOEmpty + 2,
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
// a_desc / b_desc describe the K2 pair and the Q tile at their first byte;
// each K = 16 step advances the start address (in 16-byte units) inside the
// 128-byte swizzle atom, and by one 64-column region every 4 steps.
template <int D>
__device__ __forceinline__ void issue_score_desc(uint32_t tmem_d, uint64_t a_desc, uint64_t b_desc) {
  constexpr uint32_t idesc = make_idesc_bf16(128, 64, false, false);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint64_t a = a_desc + (uint64_t)((k_slot_off<D>(kk / 4, 0) + (kk % 4) * 32) >> 4);
    const uint64_t b = b_desc + (uint64_t)(((kk / 4) * 8192 + (kk % 4) * 32) >> 4);
    umma_bf16(tmem_d, a, b, idesc, kk > 0 ? 1u : 0u);
  }
}

// O^T[128][64] (+)= V2^T . P^T: M = 128 head-dim rows, N = 64 query rows,
// K = 128 key rows.  Both operands MN-major; each K = 16 step moves 16 key
// rows (2 KB) down.  The second 64-row atom of A (head dims 64..127) sits
// 8 KB after the first (LBO).  For D = 64 that atom is other, in-bounds
// shared memory: TMEM lanes 64..127 then hold values that no one reads (row m
// of the product depends on row m of A only).
template <int D>
__device__ __forceinline__ void issue_pv_desc(uint32_t tmem_o, uint64_t a_desc, uint64_t b_desc,
                                              bool accumulate) {
  constexpr uint32_t idesc = make_idesc_bf16(128, 64, true, true);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const uint64_t a = a_desc + (uint64_t)((v_slot_off<D>(kk / 4, 0) + (kk % 4) * 2048) >> 4);
    const uint64_t b = b_desc + (uint64_t)((kk * 2048) >> 4);
    umma_bf16(tmem_o, a, b, idesc, (accumulate || kk > 0) ? 1u : 0u);
  }
}

template <int D>
__device__ __forceinline__ void issue_score_mma(uint32_t tmem_d, uint32_t k_base, uint32_t q_base) {
  issue_score_desc<D>(tmem_d, make_sdesc_sw128(k_base, 16u, 1024u), make_sdesc_sw128(q_base, 16u, 1024u));
}
template <int D>
__device__ __forceinline__ void issue_pv_mma(uint32_t tmem_o, uint32_t v_base, uint32_t p_base,
                                             bool accumulate) {
  issue_pv_desc<D>(tmem_o, make_sdesc_sw128(v_base, 8192u, 1024u),
                   make_sdesc_sw128(p_base, 8192u, 1024u), accumulate);
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
// The first barrier also ORs the warps' abort flags: if any warp of the group
// gave up a wait, every warp returns true there (and nothing is reduced), so
// the group leaves its loop together instead of leaving a warp behind at a
// barrier that the others never reach.
template <bool IsMax>
__device__ __forceinline__ bool col_reduce32(const float (&v)[32], float* red, float* fin, int wq,
                                             int lane, int t128, uint32_t bar_id, bool aborted) {
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
  if (bar_red_or(bar_id, 128, aborted)) return true;
  if (t128 < 32) {
    fin[t128] = red_op<IsMax>(red_op<IsMax>(red[t128], red[32 + t128]),
                              red_op<IsMax>(red[64 + t128], red[96 + t128]));
  }
  named_barrier_sync(bar_id, 128);
  return false;
}

// Probabilities of one key row for 32 query columns: p = 2^x (0 for a
// masked row), added to the row-sum partials and packed as bf16 pairs.  Three
// column pairs in eight take the FMA-pipe exponential, the rest the MUFU one,
// which balances the two units.
// CLAMP = false where the offsets are known to be >= -120 (see kNoClampBound).
template <bool CLAMP>
__device__ __forceinline__ void compute_probs(const uint32_t (&x)[32], bool valid, float (&lp)[32],
                                              uint32_t (&pk)[16]) {
  if (valid) {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const float x0 = __uint_as_float(x[2 * j]), x1 = __uint_as_float(x[2 * j + 1]);
      const uint64_t pp = ((j & 7) < VSA_POLY8) ? exp2_fma2_t<CLAMP>(x0, x1) : pk2(fast_exp2(x0), fast_exp2(x1));
      upk2(fadd2(pk2(lp[2 * j], lp[2 * j + 1]), pp), lp[2 * j], lp[2 * j + 1]);
      float p0, p1;
      upk2(pp, p0, p1);
      pk[j] = pack_bf16x2(p0, p1);
    }
  } else {
#pragma unroll
    for (int j = 0; j < 16; ++j) pk[j] = 0u;
  }
}

// This key row's half of the swizzled P^T tile.
__device__ __forceinline__ void store_probs(const uint32_t (&pk)[16], uint8_t* pbuf, int row, int grp) {
#pragma unroll
  for (int ch = 0; ch < 4; ++ch) {
    *reinterpret_cast<uint4*>(pbuf + sw128_off(row, 4 * grp + ch)) =
        make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
  }
}

// The rare step of the online softmax (a logit more than kOffsetLimit above
// the running maximum of its column, log2 units, after an item's first step): the exact
// column maxima over this step's valid key rows, the new running maxima
// (published in mns), the factors 2^(old - new) (in asc) and O^T rescaled by
// them once the PV products so far are done.  Out of line so that its
// registers do not weigh on the common path.  Returns false when the group
// agreed to abort (some warp had given up a wait); a wait given up here sets
// `aborted`, which the group's next barrier reports.
__device__ __noinline__ bool rescale_step(uint32_t t_s0, uint32_t t_s1, bool two, bool valid0,
                                          bool valid1, float c, float* red, float* fin,
                                          float* mns, float* asc, int wq, int lane, int t128,
                                          uint32_t bar_red, uint64_t* pempty, uint32_t pparity,
                                          uint32_t t_o, bool& aborted, volatile int* abort_flag,
                                          int* status) {
  {
    uint32_t x[32];
    float masked[32];
    tmem_ld32(t_s0, x);
#pragma unroll
    for (int q = 0; q < 32; ++q) masked[q] = valid0 ? __uint_as_float(x[q]) * c : -INFINITY;
    if (two) {
      tmem_ld32(t_s1, x);
#pragma unroll
      for (int q = 0; q < 32; ++q) masked[q] = fmaxf(masked[q], valid1 ? __uint_as_float(x[q]) * c : -INFINITY);
    }
    if (col_reduce32<true>(masked, red, fin, wq, lane, t128, bar_red, aborted)) return false;
  }
  if (t128 < 32) {
    const float old = -mns[t128];
    const float nm = fmaxf(old, fin[t128]);
    asc[t128] = fast_exp2(old - nm);
    mns[t128] = -nm;
  }
  named_barrier_sync(bar_red, 128);
  if (!aborted && !warp_wait(pempty, pparity, abort_flag, status)) aborted = true;
  tc_fence_after_sync();
  uint32_t ov[32];
  tmem_ld32(t_o, ov);
#pragma unroll
  for (int q = 0; q < 32; ++q) ov[q] = __float_as_uint(__uint_as_float(ov[q]) * asc[q]);
  tmem_st32(t_o, ov);
  return true;
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

// A 64 x 64 tile of a strided [B, H, S, D] view through its 4-D tensor map:
// head dims d0 .. d0+63 of sequence slots s .. s+63 of (b, h).  Slots past the
// view's end arrive as zeros.
__device__ __forceinline__ void load_view_tile(void* dst, const CUtensorMap* map, TmaAxes ax,
                                               uint64_t* bar, int d0, int s, int h, int b,
                                               uint64_t hint) {
  const int c1 = ax.s == 1 ? s : (ax.h == 1 ? h : b);
  const int c2 = ax.s == 2 ? s : (ax.h == 2 ? h : b);
  const int c3 = ax.s == 3 ? s : (ax.h == 3 ? h : b);
  tma_load_4d(dst, map, bar, d0, c1, c2, c3, hint);
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
  float* inv_l = reinterpret_cast<float*>(smem + L::kInvLOff);
  float* lse_s = reinterpret_cast<float*>(smem + L::kLseOff);
  int2* kmeta = reinterpret_cast<int2*>(smem + L::kKMetaOff);
  int2* smeta = reinterpret_cast<int2*>(smem + L::kSMetaOff);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);

  const int tid = threadIdx.x;
  const int warp = tid / 32, lane = tid % 32;
  const long long n_items = (long long)p.B * p.H * p.nq;
  const long long it0 = blockIdx.x, it_step = gridDim.x;

  if (tid == 0) {
    for (int i = 0; i < L::kNumBars; ++i) {
      uint32_t count = 1;  // TMA transaction arrival or one tcgen05.commit
      if ((i >= L::kSEmpty && i < L::kSEmpty + kNS) || (i >= L::kPFull && i < L::kPFull + kNP) ||
          i == L::kLFull || i == L::kLFull + 1)
        count = 8;  // one arrival per softmax warp
      if (i >= L::kSFull && i < L::kSFull + kNS) count = 2;
      if (i == L::kOEmpty || i == L::kOEmpty + 1) count = 4;   // epilogue warps
      mbar_init(bars + i, count);
    }
    *abort_flag = 0;
    *reinterpret_cast<volatile int*>(smem + L::kVIssuedOff) = 0;
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

  // Register split by warpgroup: producers/MMA and the epilogue give
  // registers to the two softmax warpgroups.  The launch reserves 128 per
  // thread (512 x 128 = 65536); the split needs 128 x (64 + 192 + 192 + 64).
  if (warp < 4) {
    regs_dec<kRegsProducer>();
    if (warp == 0 || warp == 2) {
      // ===================== producers (whole warp) =====================
      const bool is_k = (warp == 0);
      const uint64_t pol_q = l2_policy_evict_first();
      const uint64_t pol_kv = l2_policy_evict_last();
      uint32_t gp = 0;  // pair counter over this CTA's items (32 bits: power-of-two ring math)
      bool ok = true;
      uint32_t n = 0;
      for (long long it = it0; ok && it < n_items; it += it_step, ++n) {
        const Item x = load_item(p, it);
        if (is_k) {
          if (lane == 0) {
            check_item(p, it);
            if (n >= 1)
              ok = mbar_wait(bars + L::kQEmpty, (uint32_t)((n - 1) & 1), abort_flag, p.status);
            if (ok) {
              mbar_arrive_expect_tx(bars + L::kQFull, L::kQ);
#pragma unroll
              for (int dh = 0; dh < L::DH; ++dh)
                load_view_tile(smem + L::kQOff + dh * 8192, &tm_q, p.q_ax, bars + L::kQFull, dh * 64,
                               (int)x.q_tok, x.h, x.b, pol_q);
            }
          }
          ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        }
        const int32_t* idx_row = p.q2k_idx + (x.group * p.nq + x.a) * (long long)p.idx_stride;
        const int np = (x.num + 1) / 2;
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
              const int N = is_k ? L::NK : L::NV;
              const int st = (int)(gp % (uint32_t)N);
              const uint32_t u = gp / (uint32_t)N;
              // One TMA engine serves both producers in request order: K of
              // pair g waits until V of pair g - kKLead has been requested, so
              // K requests for far-ahead pairs never queue in front of V
              // requests that are needed sooner.
              if (is_k && gp >= kKLead)
                ok = spin_until_at_least(reinterpret_cast<volatile int*>(smem + L::kVIssuedOff),
                                         (int)(gp - kKLead + 1), abort_flag, p.status);
              if (ok && u >= 1)
                ok = mbar_wait(bars + (is_k ? L::kKEmpty : L::kVEmpty) + st, (uint32_t)((u - 1) & 1),
                               abort_flag, p.status);
              if (ok) {
                uint64_t* full = bars + (is_k ? L::kKFull : L::kVFull) + st;
                if (is_k) {
                  kmeta[st] = make_int2(l0, l1);
                  uint8_t* dst = smem + L::kKOff + st * L::kK2;
                  mbar_arrive_expect_tx(full, L::kK2);
#pragma unroll
                  for (int dh = 0; dh < L::DH; ++dh) {
                    load_view_tile(dst + k_slot_off<D>(dh, 0), &tm_k, p.k_ax, full, dh * 64, r0, x.h, x.b, pol_kv);
                    load_view_tile(dst + k_slot_off<D>(dh, 1), &tm_k, p.k_ax, full, dh * 64, r1, x.h, x.b, pol_kv);
                  }
                } else {
                  uint8_t* dst = smem + L::kVOff + st * L::kV2;
                  mbar_arrive_expect_tx(full, L::kV2);
#pragma unroll
                  for (int dh = 0; dh < L::DH; ++dh) {
                    load_view_tile(dst + v_slot_off<D>(0, dh), &tm_v, p.v_ax, full, dh * 64, r0, x.h, x.b, pol_kv);
                    load_view_tile(dst + v_slot_off<D>(1, dh), &tm_v, p.v_ax, full, dh * 64, r1, x.h, x.b, pol_kv);
                  }
                  *reinterpret_cast<volatile int*>(smem + L::kVIssuedOff) = (int)(gp + 1);
                }
              }
            }
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!ok) break;
            ++gp;
          }
        }
      }
      // drain: every stage's release (a tcgen05 commit) lands before exit
      if (ok && lane == 0) {
        const int N = is_k ? L::NK : L::NV;
        for (uint32_t g = (gp > (uint32_t)N ? gp - N : 0u); g < gp; ++g) {
          if (!mbar_wait(bars + (is_k ? L::kKEmpty : L::kVEmpty) + (int)(g % N),
                         (uint32_t)((g / N) & 1), abort_flag, p.status))
            break;
        }
      }
      __syncwarp();
    } else if (warp == 1) {
      // ===================== score products S^T = K2 . Q^T =====================
      const uint64_t desc_k = make_sdesc_sw128(sbase + L::kKOff, 16u, 1024u);
      const uint64_t desc_q = make_sdesc_sw128(sbase + L::kQOff, 16u, 1024u);
      uint32_t gp = 0, n = 0, n_mine = 0;
      for (long long it = it0; it < n_items; it += it_step) ++n_mine;
      bool ok = true;
      for (long long it = it0; ok && it < n_items; it += it_step, ++n) {
        const Item x = load_item(p, it);
        const int np = (x.num + 1) / 2;
        if (!warp_wait(bars + L::kQFull, (uint32_t)(n & 1), abort_flag, p.status)) { ok = false; break; }
        for (int i = 0; i < np; ++i, ++gp) {
          const int sb = (int)(gp % kNS);
          const int ks = (int)(gp % L::NK);
          if (!warp_wait(bars + L::kKFull + ks, (uint32_t)((gp / L::NK) & 1), abort_flag, p.status)) { ok = false; break; }
          if (gp >= kNS && !warp_wait(bars + L::kSEmpty + sb, (uint32_t)((gp / kNS - 1) & 1), abort_flag, p.status)) { ok = false; break; }
          if (lane == 0) smeta[sb] = kmeta[ks];
          __syncwarp();
          tc_fence_after_sync();
          if (elect_one()) {
            issue_score_desc<D>(tmem_base + 64u * sb, desc_k + (uint64_t)((ks * L::kK2) >> 4), desc_q);
            umma_commit(bars + L::kSFull + sb);
            umma_commit(bars + L::kKEmpty + ks);
            if (i == np - 1 && n + 1 < n_mine) umma_commit(bars + L::kQEmpty);
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(bars + L::kSFull + sb);
        }
        if (!ok) break;
        if (np == 0 && n + 1 < n_mine) {
          // no products for this item: release its Q tile at once
          if (elect_one()) umma_commit(bars + L::kQEmpty);
          __syncwarp();
        }
      }
    } else {
      // ===================== PV products O^T += V2^T . P^T =====================
      const uint64_t desc_v = make_sdesc_sw128(sbase + L::kVOff, 8192u, 1024u);
      const uint64_t desc_p = make_sdesc_sw128(sbase + L::kPOff, 8192u, 1024u);
      uint32_t gp = 0, n = 0;
      bool ok = true;
      for (long long it = it0; ok && it < n_items; it += it_step, ++n) {
        const Item x = load_item(p, it);
        const int o = (int)(n & 1);
        const int np = (x.num + 1) / 2;
        // the epilogue of item n - 2 must have read this output buffer
        if (n >= 2 && !warp_wait(bars + L::kOEmpty + o, (uint32_t)(((n - 2) >> 1) & 1), abort_flag, p.status)) { ok = false; break; }
        for (int i = 0; i < np; ++i, ++gp) {
          const int vs = (int)(gp % L::NV);
          const int pb = (int)(gp % kNP);
          if (!warp_wait(bars + L::kVFull + vs, (uint32_t)((gp / L::NV) & 1), abort_flag, p.status)) { ok = false; break; }
          if (!warp_wait(bars + L::kPFull + pb, (uint32_t)((gp / kNP) & 1), abort_flag, p.status)) { ok = false; break; }
          tc_fence_after_sync();
          if (elect_one()) {
            issue_pv_desc<D>(tmem_base + kTmemO + 64u * o, desc_v + (uint64_t)((vs * L::kV2) >> 4),
                             desc_p + (uint64_t)((pb * L::kP) >> 4), i > 0);
            umma_commit(bars + L::kPEmpty + pb);
            umma_commit(bars + L::kVEmpty + vs);
            if (i == np - 1) umma_commit(bars + L::kOFull + o);
          }
          __syncwarp();
        }
        if (!ok) break;
        if (np == 0) {
          // empty selection: hand the output buffer over in order anyway
          if (elect_one()) umma_commit(bars + L::kOFull + o);
          __syncwarp();
        }
      }
    }
  } else if (warp < 12) {
    regs_inc<kRegsSoftmax>();
    // ===================== softmax (two groups of 4 warps) =====================
    const int grp = (warp - 4) / 4;              // query columns 32*grp .. 32*grp+31
    const int wq = warp & 3;                     // TMEM lane quarter
    const int t128 = (warp - 4 - 4 * grp) * 32 + lane;
    const int Lr = wq * 32 + lane;               // TMEM lane: key row of S^T, head dim of O^T
    const int half = Lr >> 6, r = Lr & 63;
    const uint32_t col0 = 32u * grp;
    const uint32_t t_lane = tmem_base + (uint32_t(wq * 32) << 16);
    const uint32_t bar_vote = 1 + 2 * grp, bar_red = 2 + 2 * grp;
    float* red = red_all + grp * 128;
    float* fin = fin_all + col0;
    float* asc = reinterpret_cast<float*>(smem + L::kAlphaOff) + col0;
    const float c = p.scale_log2;
    uint32_t gp = 0, n = 0;
    bool ok = true;
    // A wait that gives up only sets `aborted` (this warp then skips its later
    // waits); the group's next barrier ORs the flag, and there every warp of
    // the group leaves the loop together (see col_reduce32).
    bool aborted = false;
    auto wwait = [&](uint64_t* bar, uint32_t parity) {
      if (!aborted && !warp_wait(bar, parity, abort_flag, p.status)) aborted = true;
    };
    // minus the running max per query column (log2 units): the same for all
    // threads of the group, so it lives in shared memory and is read as
    // broadcast 16-byte loads (it changes only at a rescale)
    float* mns = reinterpret_cast<float*>(smem + L::kMnOff) + col0;
    if (t128 < 32) mns[t128] = 0.f;
    named_barrier_sync(bar_red, 128);
    const uint64_t cc = pk2(c, c);
    for (long long it = it0; ok && it < n_items; it += it_step, ++n) {
      const Item x = load_item(p, it);
      const int o = (int)(n & 1);
      const int np = (x.num + 1) / 2;
      // bound on every logit of the item (log2 units); infinite without one
      const float qk_bound = p.qk_bound ? p.qk_bound[x.group * p.nq + x.a] : INFINITY;
      bool novote = false;  // set by the item's first step
      float lp[32];
#pragma unroll
      for (int q = 0; q < 32; ++q) lp[q] = 0.f;
      if (qk_bound <= kNoClampBound) {
        // the bound itself is every column's reference max: each offset
        // s*c - m is then in [-2 * bound, 0], so no step needs the exact
        // maximum, a vote or the exponential's clamp (same results up to
        // rounding: the probabilities of a column share one scale factor)
        if (t128 < 32) mns[t128] = -qk_bound;
        if (bar_red_or(bar_red, 128, aborted)) { ok = false; break; }
        novote = true;
      }
      // One step: two pairs (the second may be absent at the end of an
      // item), so the fixed cost of the handshakes is paid once per 4 KV
      // tiles.  The step is compiled for two pairs with the overflow vote, for
      // one pair with it, and for two pairs without it (later steps of an item
      // whose bound rules a refresh out), so that the common step carries no
      // run-time tests of the pair count.  (A further copy for two pairs of
      // full blocks, free of the masked key-row tests, ran slower:
      // instruction-cache pressure.)
      auto step = [&](int i, auto two_tag, auto vote_tag) -> bool {
        constexpr bool two = decltype(two_tag)::value;
        constexpr bool vote = decltype(vote_tag)::value;
        const uint32_t g0 = gp, g1 = gp + 1;
        bool valid0, valid1 = false;
        // S^T of pair g1 is committed after that of g0 by the same thread, so
        // its barrier covers both products (and both key-count records)
        {
          const uint32_t gl = two ? g1 : g0;
          wwait(bars + L::kSFull + (int)(gl % kNS), (uint32_t)((gl / kNS) & 1));
        }
        {
          const int2 l0 = smeta[g0 % kNS];
          valid0 = r < (half ? l0.y : l0.x);
          if (two) {
            const int2 l1 = smeta[g1 % kNS];
            valid1 = r < (half ? l1.y : l1.x);
          }
        }
        const uint32_t s0_col = 64u * (uint32_t)(g0 % kNS) + col0;
        const uint32_t s1_col = 64u * (uint32_t)(g1 % kNS) + col0;
        tc_fence_after_sync();
        uint32_t x0[32], x1[32];                 // logits, then log2-domain offsets
        VSA_TMEM_LD16(t_lane + s0_col, x0, 0);
        VSA_TMEM_LD16(t_lane + s0_col + 16u, x0, 16);
        if (two) {
          VSA_TMEM_LD16(t_lane + s1_col, x1, 0);
          VSA_TMEM_LD16(t_lane + s1_col + 16u, x1, 16);
        }
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
        if (vote && i == 0) {
          // an item's first step: the running max starts as the exact column
          // max over this step's valid key rows (x0 is loaded again after)
          float fm[32];
#pragma unroll
          for (int q = 0; q < 32; ++q) {
            const float a = valid0 ? __uint_as_float(x0[q]) * c : -INFINITY;
            const float b = valid1 ? __uint_as_float(x1[q]) * c : -INFINITY;
            fm[q] = fmaxf(a, b);
          }
          if (col_reduce32<true>(fm, red, fin, wq, lane, t128, bar_red, aborted)) return false;
          // later offsets are at most bound - max: if that is within the
          // limit for every column of the group, later steps need no vote
          bool fits = true;
          if (t128 < 32) {
            const float mn = (fin[t128] == -INFINITY) ? 0.f : -fin[t128];
            mns[t128] = mn;
            fits = qk_bound + mn <= kOffsetLimit && qk_bound <= kNoClampBound;
          }
          novote = bar_red_and(bar_red, 128, fits);
          VSA_TMEM_LD16(t_lane + s0_col, x0, 0);
          VSA_TMEM_LD16(t_lane + s0_col + 16u, x0, 16);
          asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
        }
        bool rescale = false;
        {
          // offsets s * c - m, two columns per instruction
          float w0 = -INFINITY, w1 = -INFINITY;
          const ulonglong2* mn2 = reinterpret_cast<const ulonglong2*>(mns);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const ulonglong2 mm = mn2[j / 2];
            const uint64_t nm = (j & 1) ? mm.y : mm.x;
            float a, b;
            upk2(ffma2(pk2(__uint_as_float(x0[2 * j]), __uint_as_float(x0[2 * j + 1])), cc, nm), a, b);
            x0[2 * j] = __float_as_uint(a);
            x0[2 * j + 1] = __float_as_uint(b);
            if (vote) w0 = fmax3(w0, a, b);
            if (two) {
              upk2(ffma2(pk2(__uint_as_float(x1[2 * j]), __uint_as_float(x1[2 * j + 1])), cc, nm), a, b);
              x1[2 * j] = __float_as_uint(a);
              x1[2 * j + 1] = __float_as_uint(b);
              if (vote) w1 = fmax3(w1, a, b);
            }
          }
          const float worst = fmaxf(valid0 ? w0 : -INFINITY, valid1 ? w1 : -INFINITY);
          // does any logit exceed the running max by more than the limit?
          if (vote && i > 0 && bar_red_or(bar_vote, 128, aborted || worst > kOffsetLimit)) {
            // rare: a refresh, or some warp of the group gave up a wait
            if (bar_red_or(bar_vote, 128, aborted)) return false;
            rescale = true;
          }
        }
        if (vote && rescale) {
          // rare step, out of line: new running maxima (shared memory), the
          // factors 2^(old - new) (asc) and O^T rescaled; the partial sums
          // and the offsets are brought up to date here
          const uint32_t gq = g0 - 1;
          if (!rescale_step(t_lane + s0_col, t_lane + s1_col, two, valid0, valid1, c, red, fin, mns,
                            asc, wq, lane, t128, bar_red, bars + L::kPEmpty + (int)(gq % kNP),
                            (uint32_t)((gq / kNP) & 1), t_lane + kTmemO + 64u * o + col0, aborted,
                            abort_flag, p.status)) return false;
#pragma unroll
          for (int q = 0; q < 32; ++q) lp[q] *= asc[q];
          tmem_ld32(t_lane + s0_col, x0);
          if (two) tmem_ld32(t_lane + s1_col, x1);
#pragma unroll
          for (int q = 0; q < 32; ++q) {
            const float mq = mns[q];
            x0[q] = __float_as_uint(fmaf(__uint_as_float(x0[q]), c, mq));
            x1[q] = two ? __float_as_uint(fmaf(__uint_as_float(x1[q]), c, mq)) : __float_as_uint(-INFINITY);
          }
        }
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(bars + L::kSEmpty + (int)(g0 % kNS));
          if (two) mbar_arrive(bars + L::kSEmpty + (int)(g1 % kNS));
        }
        // the exponentials first, so that they overlap the PV products still
        // reading the P^T buffers
        uint32_t pk0[16], pk1[16];
        compute_probs<vote>(x0, valid0, lp, pk0);
        if (two) compute_probs<vote>(x1, valid1, lp, pk1);
        // the P^T buffers are free once the PV products of pairs g0 - kNP and
        // g0 + 1 - kNP are done; both are committed by one thread in order, so
        // the barrier of the later one covers both
        if (g0 + 1 >= kNP) {
          const uint32_t gq = g0 + 1 - kNP;
          wwait(bars + L::kPEmpty + (int)(gq % kNP), (uint32_t)((gq / kNP) & 1));
        }
        store_probs(pk0, smem + L::kPOff + (int)(g0 % kNP) * L::kP, Lr, grp);
        if (two) store_probs(pk1, smem + L::kPOff + (int)(g1 % kNP) * L::kP, Lr, grp);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(bars + L::kPFull + (int)(g0 % kNP));
          if (two) mbar_arrive(bars + L::kPFull + (int)(g1 % kNP));
        }
        gp += two ? 2 : 1;
        return true;
      };
      for (int i = 0; i < np; i += 2) {
        bool more;
        if (i + 1 >= np) more = step(i, BoolTag<false>{}, BoolTag<true>{});
        else if (novote) more = step(i, BoolTag<true>{}, BoolTag<false>{});
        else more = step(i, BoolTag<true>{}, BoolTag<true>{});
        if (!more) { ok = false; break; }
      }
      if (!ok) break;
      // end of item: 1 / row sums for the epilogue
      if (n >= 2) wwait(bars + L::kOEmpty + o, (uint32_t)(((n - 2) >> 1) & 1));
      if (col_reduce32<false>(lp, red, fin, wq, lane, t128, bar_red, aborted)) { ok = false; break; }
      if (t128 < 32) {
        const float l = fin[t128];
        inv_l[o * 64 + col0 + t128] = l > 0.f ? 1.f / l : 0.f;
        // log2 of the column's sum of 2^(s*c) = running max + log2(sum)
        lse_s[o * 64 + col0 + t128] = l > 0.f ? __log2f(l) - mns[t128] : -INFINITY;
      }
      named_barrier_sync(bar_red, 128);
      __syncwarp();
      if (lane == 0) mbar_arrive(bars + L::kLFull + o);
    }
    // drain: the last PV products' releases of the P^T buffers land before exit
    if (ok && !aborted) {
      for (uint32_t g = (gp > (uint32_t)kNP ? gp - kNP : 0u); g < gp; ++g) {
        if (!warp_wait(bars + L::kPEmpty + (int)(g % kNP), (uint32_t)((g / kNP) & 1), abort_flag, p.status)) break;
      }
    }
  } else {
    regs_dec<kRegsEpilogue>();
    // ===================== epilogue =====================
    // O^T / l leaves TMEM (lane = head dim) in 16-row slices through a small
    // fp32 tile, so the combine and the global traffic run in row order with
    // 8-byte loads and stores.
    const int wq = warp & 3;
    const int d = wq * 32 + lane;                // TMEM lane = head dim of O^T
    const int t128 = (warp - 12) * 32 + lane;
    const uint32_t t_lane = tmem_base + (uint32_t(wq * 32) << 16);
    const bool active = wq * 32 < D;
    float* stage = reinterpret_cast<float*>(smem + L::kStageOff);   // [16][D]
    constexpr int kChunks = 16 * D / 4;                             // 4-float chunks per slice
    constexpr int kPerThread = kChunks / 128;
    const int d0 = (t128 % (D / 4)) * 4;                            // fixed per thread
    uint32_t n = 0;
    for (long long it = it0; it < n_items; it += it_step, ++n) {
      const Item x = load_item(p, it);
      const int o = (int)(n & 1);
      // the four warps agree before their first named barrier of the item,
      // so a warp that gave up a wait never leaves the others at one
      bool bad = !warp_wait(bars + L::kOFull + o, (uint32_t)((n >> 1) & 1), abort_flag, p.status);
      if (!bad) bad = !warp_wait(bars + L::kLFull + o, (uint32_t)((n >> 1) & 1), abort_flag, p.status);
      if (bar_red_or(5, 128, bad)) break;
      if (p.lse && t128 < 64) {
        // natural-log log-sum-exp of each real query row (0 on padding rows)
        const int q = t128;
        if (q < x.q_len)
          p.lse[x.group * p.lse_seq + x.q_tok + q] = lse_s[o * 64 + q] * 0.69314718055994531f;
        else if (!p.varlen)
          p.lse[x.group * p.lse_seq + x.q_tok + q] = 0.f;
      }
      float4 oc = make_float4(0.f, 0.f, 0.f, 0.f);
      if (COMBINE) oc = *reinterpret_cast<const float4*>(p.out_c + (x.group * p.nq + x.a) * (long long)D + d0);
      // element offsets of the block's first token in out and gate
      __nv_bfloat16* orow0 = p.out + x.b * p.out_st.b + x.h * p.out_st.h + x.q_tok * p.out_st.s + d0;
      const __nv_bfloat16* grow0 =
          GATED ? p.gate + x.b * p.gate_st.b + x.h * p.gate_st.h + x.q_tok * p.gate_st.s + d0 : nullptr;
      for (int rnd = 0; rnd < 4; ++rnd) {
        if (active) {
          uint32_t ov[16];
          if (x.num > 0) {
            tc_fence_after_sync();
            VSA_TMEM_LD16(t_lane + kTmemO + 64u * o + 16u * rnd, ov, 0);
            asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
          } else {
#pragma unroll
            for (int q = 0; q < 16; ++q) ov[q] = 0u;
          }
#pragma unroll
          for (int q = 0; q < 16; ++q)
            stage[q * D + d] = __uint_as_float(ov[q]) * inv_l[o * 64 + 16 * rnd + q];
        }
        if (rnd == 3) {
          // output buffer and 1/l of this item fully read: hand them back
          tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive(bars + L::kOEmpty + o);
        }
        named_barrier_sync(5, 128);
#pragma unroll
        for (int k = 0; k < kPerThread; ++k) {
          const int c = t128 + 128 * k;
          const int row = c / (D / 4);
          const int q = 16 * rnd + row;
          if (q < x.q_len) {
            const float4 v4 = *reinterpret_cast<const float4*>(stage + row * D + d0);
            float v0 = v4.x, v1 = v4.y, v2 = v4.z, v3 = v4.w;
            if (COMBINE) {
              if (GATED) {
                const uint2 graw = *reinterpret_cast<const uint2*>(grow0 + q * p.gate_st.s);
                const float2 g01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&graw.x));
                const float2 g23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&graw.y));
                v0 = fmaf(oc.x, g01.x, v0);
                v1 = fmaf(oc.y, g01.y, v1);
                v2 = fmaf(oc.z, g23.x, v2);
                v3 = fmaf(oc.w, g23.y, v3);
              } else {
                v0 += oc.x; v1 += oc.y; v2 += oc.z; v3 += oc.w;
              }
            }
            *reinterpret_cast<uint2*>(orow0 + q * p.out_st.s) =
                make_uint2(pack_bf16x2(v0, v1), pack_bf16x2(v2, v3));
          } else if (!p.varlen) {
            *reinterpret_cast<uint2*>(orow0 + q * p.out_st.s) = make_uint2(0u, 0u);
          }
        }
        named_barrier_sync(5, 128);
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

// Self-test of the FMA-pipe exponential: y[i] = exp2_fma2(x[i]) (the lower
// half of the pair; the upper half gets x[i] too and must agree).
__global__ void selftest_exp2_kernel(const float* x, float* y, long long n, int* mismatch) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  float lo, hi;
  upk2(exp2_fma2(x[i], x[i]), lo, hi);
  y[i] = lo;
  if (__float_as_uint(lo) != __float_as_uint(hi)) atomicAdd(mismatch, 1);
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
EncodeTiledFn get_encode_fn() {
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

// 4-D map of a strided [B, H, S, D] bf16 view: dimension 0 is the head dim,
// dimensions 1..3 the sequence, head and batch axes in increasing stride
// order (an axis of extent 1 goes last, with the stride an outer contiguous
// axis would have); boxes of 64 head dims x box_rows slots of one head and
// batch, 128-byte swizzle.  The caller checked that every stride
// is a multiple of 8 elements (16 bytes) and the base 16-byte aligned.
bool make_view_map_rows(CUtensorMap* map, TmaAxes* ax, const void* base, int D, long long S,
                        int H, int B, Strides3 st, int box_rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  struct A { int id; long long ext, str; } a[3] = {{0, S, st.s}, {1, H, st.h}, {2, B, st.b}};
  // order: axes of extent > 1 by stride, then the rest
  for (int i = 0; i < 3; ++i)
    for (int j = i + 1; j < 3; ++j) {
      const bool ai = a[i].ext > 1, aj = a[j].ext > 1;
      if ((!ai && aj) || (ai == aj && ai && a[j].str < a[i].str)) { A t = a[i]; a[i] = a[j]; a[j] = t; }
    }
  cuuint64_t dims[4] = {(cuuint64_t)D, 0, 0, 0};
  cuuint64_t strides[3];
  long long outer = (long long)D * 2;  // bytes spanned so far
  for (int i = 0; i < 3; ++i) {
    long long sb = a[i].str * 2;
    if (a[i].ext <= 1 || sb <= 0) sb = outer;  // never stepped: any valid stride
    dims[i + 1] = (cuuint64_t)a[i].ext;
    strides[i] = (cuuint64_t)sb;
    outer = sb * a[i].ext > outer ? sb * a[i].ext : outer;
    const int slot = i + 1;
    if (a[i].id == 0) ax->s = slot;
    else if (a[i].id == 1) ax->h = slot;
    else ax->b = slot;
  }
  cuuint32_t box[4] = {64, 1, 1, 1};
  box[ax->s] = (cuuint32_t)box_rows;
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides,
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
  // The warpgroup register split assumes 128 registers per thread at launch;
  // with fewer, a warpgroup's register increase could never be granted.
  static int regs_ok = -1;
  if (regs_ok < 0) {
    cudaFuncAttributes attr;
    regs_ok = (cudaFuncGetAttributes(&attr, kern) == cudaSuccess && attr.numRegs == 128) ? 1 : 0;
  }
  if (!regs_ok) return VSA_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::kAlloc) !=
      cudaSuccess)
    return VSA_ERR_CUDA;
  const long long n_items = (long long)p.B * p.H * p.nq;
  const long long grid = n_items < sm_count() ? n_items : sm_count();
  kern<<<(unsigned)grid, kThreads, L::kAlloc, stream>>>(mq, mk, mv, p);
  return cudaGetLastError() == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

static bool make_view_map(CUtensorMap* map, TmaAxes* ax, const void* base, int D, long long S,
                          int H, int B, Strides3 st) {
  return make_view_map_rows(map, ax, base, D, S, H, B, st, 64);
}

int launch_sparse(const SparseParams& p_in, const void* q, Strides3 q_st, long long q_seq,
                  const void* k, Strides3 k_st, const void* v, Strides3 v_st, long long kv_seq,
                  int D, bool combine, bool gated, cudaStream_t stream) {
  if (p_in.nq <= 0 || p_in.H <= 0 || p_in.B <= 0) return VSA_OK;
  if (q_seq + 64 > 0x7FFFFFFFLL || kv_seq + 64 > 0x7FFFFFFFLL)
    return VSA_ERR_UNSUPPORTED;  // TMA coordinates are 32-bit
  SparseParams p = p_in;
  CUtensorMap mq, mk, mv;
  if (!make_view_map(&mq, &p.q_ax, q, D, q_seq, p.H, p.B, q_st) ||
      !make_view_map(&mk, &p.k_ax, k, D, kv_seq, p.H, p.B, k_st) ||
      !make_view_map(&mv, &p.v_ax, v, D, kv_seq, p.H, p.B, v_st))
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

int launch_selftest_exp2(const float* x, float* y, long long n, int* mismatch,
                         cudaStream_t stream) {
  if (n <= 0) return VSA_OK;
  selftest_exp2_kernel<<<(unsigned)((n + 255) / 256), 256, 0, stream>>>(x, y, n, mismatch);
  return cudaGetLastError() == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
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
