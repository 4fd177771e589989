// Block-sparse attention over selected 128 x 128 tiles (VSA with 128-token
// blocks), with the coarse/sparse combine fused into the epilogue.
//
// What it computes: the same as the 64-token path ("[chore] release
// fastvideo-kernel 0.3.0", block_sparse_attn_from_indices; "[perf] avoid
// full-sequence materialization in VSA coarse/sparse combine", Problem /
// Change), with 128-slot blocks: the README's kernel inventory lists
// Blackwell forward kernels for 128-token VSA tiles, and release 0.3.0 the
// 128/256-token tile fastpath.
//
// How (sm_100a).  A 128-row query tile is the tensor core's native M, so no
// transposition is needed:
//   S[128 q][128 kv] = Q[128][D] . K[128][D]^T        (K-major A and B, smem)
//   O[128 q][D]     += P[128 q][128 kv] . V[128][D]     (A = P in TMEM, B = V
//                                                         MN-major in smem)
// TMEM lane = query row, so one softmax thread owns one query row: its
// running max and row sum never leave the thread.  P is written as bf16 into
// the first 64 columns of its own S buffer (the S values are in registers by
// then); the next score product into that buffer is issued after the PV
// product that reads P by the same thread, and tcgen05 MMAs issued by one
// thread execute in issue order.
//
// Persistent grid, one CTA per SM walking the work items (query block, head,
// batch) with stride gridDim.  512 threads, four warpgroups:
//   warp 0      Q tiles (double-buffered per item) and K tiles (2-stage ring)
//   warp 1      TMEM owner; issues S(j) and PV(j-1) in that order
//   warp 2      V tiles (2-stage ring)
//   warps 4-11  softmax, two warpgroups splitting each row's key columns:
//               S(j) -> P(j) and row sums.  The item's logit bound, where it
//               is at most kNoClampBound, is the row's reference max from the
//               first tile on; otherwise the row max takes a lazy refresh
//               (the reference max moves only when a logit exceeds it by more
//               than kRefresh log2 units; then O is rescaled once the PV
//               product before it is done), with the tile max exchanged
//               between the groups until the bound rules a move out
//   warps 12-15 epilogue: O / l, out = out_c * gate + o (or out_c + o, or o),
//               bf16 stores; double-buffered O lets it overlap the next item
// Every wait is bounded and reports VSA_ERR_DEVICE_TIMEOUT.  The only named
// barrier after the role split joins the two softmax groups; it also ORs
// their abort flags, so a warp that gave up a wait never leaves the others
// behind at it.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "vsa.h"
#include "vsa_device.cuh"
#include "vsa_launch.h"

namespace vsa {
namespace b128 {

constexpr int kThreads = 512;
// registers per thread of the producer / MMA, softmax and epilogue warpgroups
#ifndef VSA128_REGS_P
#define VSA128_REGS_P 48
#endif
#ifndef VSA128_REGS_S
#define VSA128_REGS_S 184
#endif
#ifndef VSA128_REGS_E
#define VSA128_REGS_E 96
#endif
constexpr uint32_t kRegsProducer = VSA128_REGS_P, kRegsSoftmax = VSA128_REGS_S,
                   kRegsEpilogue = VSA128_REGS_E;
constexpr uint32_t kLaunchRegs = 128;  // 512 x 128 = 65536
static_assert(128u * (kRegsProducer + 2u * kRegsSoftmax + kRegsEpilogue) <= 512u * kLaunchRegs,
              "register split exceeds the launch's registers");
constexpr int NK = 2, NV = 2;
// Largest excess (log2 units) of a logit over its row's reference max that
// is exponentiated without moving the reference: probabilities stay below
// 2^8, well inside bf16 and fp32 range.
constexpr float kRefresh = 8.f;
// Largest excess (log2 units) of a logit over its row's first-tile max that
// the logit bound must rule out before an item's later tiles skip the max
// exchange: probabilities then stay below 2^32 (bf16 and fp32 hold them).
constexpr float kBoundLimit = 32.f;
// Largest logit bound (log2 units) for which those tiles also skip the
// FMA-pipe exponential's lower clamp: every offset s*c - m is then >= -2 *
// bound (s*c >= -bound, the reference max m <= bound), so >= -120.
constexpr float kNoClampBound = 60.f;
#ifndef VSA128_POLY8
#define VSA128_POLY8 1  // column pairs in eight whose exponential runs on the FMA pipe
#endif

template <int D>
struct Layout {
  static constexpr int DH = D / 64;
  static constexpr uint32_t kTile = 128u * D * 2u;            // Q, K or V tile, bf16
  static constexpr uint32_t kQOff = 0;                         // [2] Q tiles
  static constexpr uint32_t kKOff = kQOff + 2 * kTile;         // [NK]
  static constexpr uint32_t kVOff = kKOff + NK * kTile;        // [NV]
  static constexpr uint32_t kInvLOff = kVOff + NV * kTile;     // [2][128] f32
  // exchange slots [4][2 halves][128] f32: tile maxima by tile parity (0, 1),
  // row sums by item parity (2, 3)
  static constexpr uint32_t kXchOff = kInvLOff + 2u * 128u * 4u;
  static constexpr uint32_t kKMetaOff = kXchOff + 4u * 256u * 4u;   // [NK] key counts
  static constexpr uint32_t kSMetaOff = kKMetaOff + 4u * NK;        // [2] key count per S buffer
  static constexpr uint32_t kBarOff = (kSMetaOff + 4u * 2u + 7u) & ~7u;
  static constexpr int kQFull = 0, kQEmpty = 2, kKFull = 4, kKEmpty = kKFull + NK,
                       kVFull = kKEmpty + NK, kVEmpty = kVFull + NV, kSFull = kVEmpty + NV,
                       kPFull = kSFull + 2, kPVDone = kPFull + 2, kOFull = kPVDone + 2,
                       kOEmpty = kOFull + 2, kLFull = kOEmpty + 2, kNumBars = kLFull + 2;
  static constexpr uint32_t kMiscOff = kBarOff + 8u * kNumBars;  // tmem address, abort flag
  static constexpr uint32_t kBytes = kMiscOff + 16u;
  static constexpr uint32_t kAlloc = kBytes + 1024u;
  static_assert(kKOff % 1024 == 0 && kVOff % 1024 == 0, "1 KB swizzle atoms");
  static_assert(kAlloc <= 227u * 1024u, "shared memory");
};

// TMEM columns: S buffers at 0 and 128 (P in the first 64 of each), O
// buffers at 256 and 256 + D.
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 256;

// S = Q . K^T: M = 128, N = 128, K = D.  Q and K tiles are
// [dh][128 rows][128 B] (128-byte swizzle); each K = 16 step moves 32 bytes
// inside the swizzle atom, and to the next 64-column slab every 4 steps.
template <int D>
__device__ __forceinline__ void issue_s(uint32_t tmem_d, uint32_t q_base, uint32_t k_base) {
  constexpr uint32_t idesc = make_idesc_bf16(128, 128, false, false);
  const uint64_t a0 = make_sdesc_sw128(q_base, 16u, 1024u);
  const uint64_t b0 = make_sdesc_sw128(k_base, 16u, 1024u);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint64_t off = (uint64_t)(((kk / 4) * 16384 + (kk % 4) * 32) >> 4);
    umma_bf16(tmem_d, a0 + off, b0 + off, idesc, kk > 0 ? 1u : 0u);
  }
}

// O (+)= P . V: M = 128, N = D, K = 128 key rows.  P (bf16) in TMEM, two
// values per 32-bit column, so each K = 16 step takes the next 8 columns; V
// is MN-major: 64-column slabs of [128 rows][128 B], 16 KB apart (LBO), a
// K = 16 step moves 16 rows (2 KB).
template <int D>
__device__ __forceinline__ void issue_pv(uint32_t tmem_o, uint32_t tmem_p, uint32_t v_base,
                                         bool accumulate) {
  constexpr uint32_t idesc = make_idesc_bf16(128, D, false, true);
  const uint64_t b0 = make_sdesc_sw128(v_base, 16384u, 1024u);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    umma_bf16_tmem_a(tmem_o, tmem_p + 8u * kk, b0 + (uint64_t)((kk * 2048) >> 4), idesc,
                     (accumulate || kk > 0) ? 1u : 0u);
  }
}

// A work item: 128 query rows.  With blocks of 128 slots (p.sub = 0) it is
// one query block and its selection, one tile per selected block.  With
// blocks of 256 slots (p.sub = 1) it is one half of a query block: the tile
// rows of the block's 256 slots split in two, each selected KV block read as
// two 128-key sub-tiles (the second empty when the block holds at most 128
// real keys), so both halves see exactly the block's selected keys.
template <bool B>
struct ClampTag {
  static constexpr bool value = B;
};

struct Item {
  int a;        // 128-row tile index in the sequence
  int ab;       // the caller's block index (a >> p.sub)
  int h, b;
  long long group;
  int num;      // 128-key tiles to process
  int q_len;    // real query rows of the tile (0 .. 128)
};

__device__ __forceinline__ long long num_items(const SparseParams& p) {
  return ((long long)p.B * p.H * p.nq) << p.sub;
}

__device__ __forceinline__ Item load_item(const SparseParams& p, long long it) {
  Item x;
  const long long per_group = (long long)p.nq << p.sub;
  x.a = (int)(it % per_group);
  x.ab = x.a >> p.sub;
  const long long t = it / per_group;
  x.h = (int)(t % p.H);
  x.b = (int)(t / p.H);
  x.group = t;
  const int num = p.q2k_num[t * p.nq + x.ab];
  x.num = (num < 0 ? 0 : (num > p.idx_stride ? p.idx_stride : num)) << p.sub;
  const int blk = 128 << p.sub;
  int ql = p.q_bs ? p.q_bs[x.ab] : blk;
  ql = ql < 1 ? 0 : (ql > blk ? blk : ql);
  ql -= 128 * (x.a & ((1 << p.sub) - 1));
  x.q_len = ql < 0 ? 0 : (ql > 128 ? 128 : ql);
  return x;
}

// A 128-slot tile (64 head dims) of a strided view through its 4-D map.
__device__ __forceinline__ void load_tile(void* dst, const CUtensorMap* map, TmaAxes ax,
                                          uint64_t* bar, int d0, int s, int h, int b,
                                          uint64_t hint) {
  const int c1 = ax.s == 1 ? s : (ax.h == 1 ? h : b);
  const int c2 = ax.s == 2 ? s : (ax.h == 2 ? h : b);
  const int c3 = ax.s == 3 ? s : (ax.h == 3 ? h : b);
  tma_load_4d(dst, map, bar, d0, c1, c2, c3, hint);
}

template <int D, bool COMBINE, bool GATED>
__global__ void __launch_bounds__(kThreads, 1)
    sparse128_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const SparseParams p) {
  using L = Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  float* inv_l = reinterpret_cast<float*>(smem + L::kInvLOff);
  int* kmeta = reinterpret_cast<int*>(smem + L::kKMetaOff);
  int* smeta = reinterpret_cast<int*>(smem + L::kSMetaOff);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);

  const int tid = threadIdx.x;
  const int warp = tid / 32, lane = tid % 32;
  const long long n_items = num_items(p);
  const long long it0 = blockIdx.x, it_step = gridDim.x;

  if (tid == 0) {
    for (int i = 0; i < L::kNumBars; ++i) {
      uint32_t count = 1;  // a TMA transaction arrival or one tcgen05.commit
      if (i == L::kPFull || i == L::kPFull + 1 || i == L::kLFull || i == L::kLFull + 1 ||
          i == L::kOEmpty || i == L::kOEmpty + 1)
        count = (i == L::kOEmpty || i == L::kOEmpty + 1) ? 4 : 8;  // per epilogue / softmax warp
      if (i == L::kSFull || i == L::kSFull + 1) count = 2;  // commit + key-count record
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

  if (warp < 4) {
    regs_dec<kRegsProducer>();
    if (warp == 0 || warp == 2) {
      // ===================== producers =====================
      const bool is_k = (warp == 0);
      const uint64_t pol_q = l2_policy_evict_first();
      const uint64_t pol_kv = l2_policy_evict_last();
      uint32_t g = 0;  // tile counter over this CTA's items
      uint32_t n = 0;
      bool ok = true;
      for (long long it = it0; ok && it < n_items; it += it_step, ++n) {
        const Item x = load_item(p, it);
        if (is_k && lane == 0) {
          const int qb = (int)(n & 1);
          if (n >= 2) ok = mbar_wait(bars + L::kQEmpty + qb, ((n - 2) >> 1) & 1, abort_flag, p.status);
          if (ok) {
            const int raw = p.q2k_num[x.group * p.nq + x.ab];
            if (raw < 0 || raw > p.idx_stride) set_status(p.status, VSA_ERR_INDEX_RANGE);
            const int ql = p.q_bs ? p.q_bs[x.ab] : (128 << p.sub);
            if (ql < 1 || ql > (128 << p.sub)) set_status(p.status, VSA_ERR_BLOCK_SIZE);
            mbar_arrive_expect_tx(bars + L::kQFull + qb, L::kTile);
#pragma unroll
            for (int dh = 0; dh < L::DH; ++dh)
              load_tile(smem + L::kQOff + qb * L::kTile + dh * 16384, &tm_q, p.q_ax,
                        bars + L::kQFull + qb, dh * 64, 128 * x.a, x.h, x.b, pol_q);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        const int32_t* idx_row = p.q2k_idx + (x.group * p.nq + x.ab) * (long long)p.idx_stride;
        const int smask = (1 << p.sub) - 1;
        for (int j = 0; ok && j < x.num; ++j, ++g) {
          if (lane == 0) {
            const int N = is_k ? NK : NV;
            const int st = (int)(g % (uint32_t)N);
            const uint32_t u = g / (uint32_t)N;
            if (u >= 1)
              ok = mbar_wait(bars + (is_k ? L::kKEmpty : L::kVEmpty) + st, (u - 1) & 1, abort_flag,
                             p.status);
            if (ok) {
              // tile j: sub-tile (j & smask) of selected block j >> sub
              const int part = j & smask;
              int c = idx_row[j >> p.sub], len = 0, row = 0;
              if (c < 0 || c >= p.nkv) {
                if (is_k && part == 0) set_status(p.status, VSA_ERR_INDEX_RANGE);
              } else {
                row = 128 * ((c << p.sub) + part);
                const int blk = 128 << p.sub;
                len = p.kv_bs ? p.kv_bs[c] : blk;
                if (len < 1 || len > blk) {
                  if (is_k && part == 0) set_status(p.status, VSA_ERR_BLOCK_SIZE);
                  len = 0;
                }
                // the sub-tile's real keys (none in a second half past the block's end)
                len -= 128 * part;
                len = len < 0 ? 0 : (len > 128 ? 128 : len);
              }
              uint64_t* full = bars + (is_k ? L::kKFull : L::kVFull) + st;
              if (is_k) kmeta[st] = len;
              uint8_t* dst = smem + (is_k ? L::kKOff : L::kVOff) + st * L::kTile;
              mbar_arrive_expect_tx(full, L::kTile);
#pragma unroll
              for (int dh = 0; dh < L::DH; ++dh)
                load_tile(dst + dh * 16384, is_k ? &tm_k : &tm_v, is_k ? p.k_ax : p.v_ax, full,
                          dh * 64, row, x.h, x.b, pol_kv);
            }
          }
          ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        }
      }
      // drain: every stage's release lands before exit
      if (ok && lane == 0) {
        const int N = is_k ? NK : NV;
        for (uint32_t t = (g > (uint32_t)N ? g - N : 0u); t < g; ++t)
          if (!mbar_wait(bars + (is_k ? L::kKEmpty : L::kVEmpty) + (int)(t % N), (t / N) & 1,
                         abort_flag, p.status))
            break;
        if (is_k) {
          for (uint32_t m = (n > 2u ? n - 2u : 0u); m < n; ++m)
            if (!mbar_wait(bars + L::kQEmpty + (int)(m & 1), (m >> 1) & 1, abort_flag, p.status))
              break;
        }
      }
      __syncwarp();
    } else if (warp == 1) {
      // ===================== MMA issue: S(j), then PV(j - 1) =====================
      uint32_t g = 0, n = 0;
      bool ok = true;
      for (long long it = it0; ok && it < n_items; it += it_step, ++n) {
        const Item x = load_item(p, it);
        const int qb = (int)(n & 1), o = (int)(n & 1);
        if (!warp_wait(bars + L::kQFull + qb, (n >> 1) & 1, abort_flag, p.status)) { ok = false; break; }
        const uint32_t q_addr = sbase + L::kQOff + qb * L::kTile;
        const uint32_t g0 = g;
        for (int j = 0; j <= x.num; ++j) {
          if (j < x.num) {
            const uint32_t t = g0 + j;
            const int ks = (int)(t % NK), sb = (int)(t & 1);
            if (!warp_wait(bars + L::kKFull + ks, (t / NK) & 1, abort_flag, p.status)) { ok = false; break; }
            if (lane == 0) smeta[sb] = kmeta[ks];
            __syncwarp();
            tc_fence_after_sync();
            if (elect_one()) {
              issue_s<D>(tmem_base + 128u * sb, q_addr, sbase + L::kKOff + ks * L::kTile);
              umma_commit(bars + L::kSFull + sb);
              umma_commit(bars + L::kKEmpty + ks);
              if (j == x.num - 1) umma_commit(bars + L::kQEmpty + qb);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bars + L::kSFull + sb);
          }
          if (j >= 1) {
            const uint32_t t = g0 + j - 1;
            const int vs = (int)(t % NV), sb = (int)(t & 1);
            if (j == 1 && n >= 2 &&
                !warp_wait(bars + L::kOEmpty + o, ((n - 2) >> 1) & 1, abort_flag, p.status)) { ok = false; break; }
            if (!warp_wait(bars + L::kPFull + sb, (t >> 1) & 1, abort_flag, p.status)) { ok = false; break; }
            if (!warp_wait(bars + L::kVFull + vs, (t / NV) & 1, abort_flag, p.status)) { ok = false; break; }
            tc_fence_after_sync();
            if (elect_one()) {
              issue_pv<D>(tmem_base + kTmemO + D * o, tmem_base + 128u * sb,
                          sbase + L::kVOff + vs * L::kTile, j > 1);
              umma_commit(bars + L::kVEmpty + vs);
              umma_commit(bars + L::kPVDone + sb);
              if (j == x.num) umma_commit(bars + L::kOFull + o);
            }
            __syncwarp();
          }
        }
        if (!ok) break;
        if (x.num == 0) {
          // nothing selected: hand the Q tile back and the (unwritten)
          // output buffer over in order
          if (n >= 2 && !warp_wait(bars + L::kOEmpty + o, ((n - 2) >> 1) & 1, abort_flag, p.status)) { ok = false; break; }
          if (elect_one()) {
            umma_commit(bars + L::kQEmpty + qb);
            umma_commit(bars + L::kOFull + o);
          }
          __syncwarp();
        }
        g += x.num;
      }
    }
  } else if (warp < 12) {
    regs_inc<kRegsSoftmax>();
    // ===================== softmax =====================
    // Two warpgroups split each query row's 128 key columns: a thread owns
    // one row (TMEM lane) and 64 columns.  The row's tile max is combined
    // through shared memory once per tile (named barrier 1, both groups), so
    // both halves move the reference max at the same tile; each half keeps a
    // partial row sum, added up at the end of the item.
    const int half = (warp - 4) >> 2;           // key columns 64*half .. 64*half + 63
    const int wq = warp & 3;
    const int row = wq * 32 + lane;             // TMEM lane = query row
    const uint32_t t_lane = tmem_base + (uint32_t(wq * 32) << 16);
    const uint32_t col0 = 64u * half;
    float* xch = reinterpret_cast<float*>(smem + L::kXchOff);  // [slot][half][row]
    const float c = p.scale_log2;
    const uint64_t cc = pk2(c, c);
    uint32_t g = 0, n = 0;
    // A wait that gives up sets `aborted`; the groups' next barrier ORs it and
    // every softmax warp leaves the loop there together.
    bool aborted = false, stop = false;
    auto wwait = [&](uint64_t* bar, uint32_t parity) {
      if (!aborted && !warp_wait(bar, parity, abort_flag, p.status)) aborted = true;
    };
    for (long long it = it0; !stop && it < n_items; it += it_step, ++n) {
      const Item x = load_item(p, it);
      const int o = (int)(n & 1);
      float m = -INFINITY;  // reference max of the row (log2 units)
      float l0 = 0.f, l1 = 0.f;
      // bound on every logit of the item (log2 units), from block row norms;
      // once the first tile has fixed the row maxima and the bound keeps
      // every later logit within kBoundLimit of them, later tiles skip the
      // max exchange (same results: the reference max would not move)
      const float qk_bound = p.qk_bound ? p.qk_bound[x.group * p.nq + x.ab] : INFINITY;
      bool novote = false;
      if (qk_bound <= kNoClampBound) {
        // the bound itself is the row's reference max: every offset s*c - m
        // is then in [-2 * bound, 0], so no tile needs the row max, its
        // exchange or the exponential's clamp (same results up to rounding:
        // the row's probabilities share one scale factor)
        m = qk_bound;
        novote = true;
      }
      for (int j = 0; j < x.num; ++j, ++g) {
        const int sb = (int)(g & 1);
        wwait(bars + L::kSFull + sb, (g >> 1) & 1);
        const int len = smeta[sb];
        tc_fence_after_sync();
        uint32_t s[64];
#pragma unroll
        for (int q = 0; q < 4; ++q) VSA_TMEM_LD16(t_lane + 128u * sb + col0 + 16u * q, s, 16 * q);
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
        const bool full = len >= 128;
        if (!full) {
          // masked key columns become -inf
#pragma unroll
          for (int q = 0; q < 64; ++q)
            if ((int)col0 + q >= len) s[q] = __float_as_uint(-INFINITY);
        }
        if (!novote) {
        float mx = -INFINITY;
#pragma unroll
        for (int q = 0; q < 64; q += 2) mx = fmax3(mx, __uint_as_float(s[q]), __uint_as_float(s[q + 1]));
        // the row's tile max over both halves
        float* xs = xch + (g & 1) * 256;
        xs[half * 128 + row] = mx;
        if (bar_red_or(1, 256, aborted)) { stop = true; break; }
        mx = fmaxf(mx, xs[(half ^ 1) * 128 + row]) * c;
        // move the reference only when this tile's max exceeds it by more
        // than kRefresh; then the partial sums and O (if any product has
        // accumulated; each half scales half of O's columns) are rescaled
        const bool move = mx > m + kRefresh;
        if (__any_sync(0xffffffffu, move)) {
          const float nm = move ? mx : m;
          const float alpha = (m == -INFINITY) ? 0.f : fast_exp2(m - nm);
          l0 *= alpha;
          l1 *= alpha;
          if (j > 0) {
            // O holds products up to PV(j - 1): wait for it, then scale
            const uint32_t t = g - 1;
            wwait(bars + L::kPVDone + (int)(t & 1), (t >> 1) & 1);
            tc_fence_after_sync();
            const uint32_t to = t_lane + kTmemO + D * o + (D / 2) * half;
#pragma unroll
            for (int q0 = 0; q0 < D / 2; q0 += 16) {
              uint32_t ov[16];
              VSA_TMEM_LD16(to + q0, ov, 0);
              asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
              for (int q = 0; q < 16; ++q) ov[q] = __float_as_uint(__uint_as_float(ov[q]) * alpha);
              VSA_TMEM_ST16(to + q0, ov, 0);
            }
            asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
          }
          m = nm;
        }
        if (j == 0) {
          // the first tile fixed the row maxima: can the bound rule out a move
          // for every row of the item?  (m = -inf fails the test)
          novote = bar_red_and(1, 256, qk_bound - m <= kBoundLimit && qk_bound <= kNoClampBound);
        }
        }
        // probabilities 2^(s*c - m) as bf16 pairs, sums in fp32
        uint32_t pk[32];
        // every key real (the common case): no per-element tests; the
        // vote-free tiles of an item skip the exponential's clamp
        auto full_tile = [&](auto clamp_tag) {
          constexpr bool CLAMP = decltype(clamp_tag)::value;
          const uint64_t nm2 = pk2(-m, -m);
#pragma unroll
          for (int q = 0; q < 32; ++q) {
            float a, b;
            upk2(ffma2(pk2(__uint_as_float(s[2 * q]), __uint_as_float(s[2 * q + 1])), cc, nm2), a, b);
            const uint64_t pp = ((q & 7) < VSA128_POLY8) ? exp2_fma2_t<CLAMP>(a, b)
                                                          : pk2(fast_exp2(a), fast_exp2(b));
            upk2(fadd2(pk2(l0, l1), pp), l0, l1);
            float p0, p1;
            upk2(pp, p0, p1);
            pk[q] = pack_bf16x2(p0, p1);
          }
        };
        if (full && novote) {
          full_tile(ClampTag<false>{});
        } else if (full) {
          full_tile(ClampTag<true>{});
        } else {
          // masked columns (s = -inf) give exactly 0; a row that has seen no
          // real key yet (m = -inf) too
          const bool none = (m == -INFINITY);
          const uint64_t nm2 = pk2(none ? 0.f : -m, none ? 0.f : -m);
#pragma unroll
          for (int q = 0; q < 32; ++q) {
            float a, b;
            upk2(ffma2(pk2(__uint_as_float(s[2 * q]), __uint_as_float(s[2 * q + 1])), cc, nm2), a, b);
            float p0 = fast_exp2(a), p1 = fast_exp2(b);
            if (none || (int)col0 + 2 * q >= len) p0 = 0.f;
            if (none || (int)col0 + 2 * q + 1 >= len) p1 = 0.f;
            upk2(fadd2(pk2(l0, l1), pk2(p0, p1)), l0, l1);
            pk[q] = pack_bf16x2(p0, p1);
          }
        }
        // P (bf16 pairs) into this half's 32 columns of the S buffer
        VSA_TMEM_ST16(t_lane + 128u * sb + (col0 >> 1), pk, 0);
        VSA_TMEM_ST16(t_lane + 128u * sb + (col0 >> 1) + 16u, pk, 16);
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(bars + L::kPFull + sb);
      }
      if (stop) break;
      // end of item: the row sum of both halves, then 1 / l for the epilogue
      // (after the epilogue of item n - 2 released this buffer)
      float* xs = xch + (2 + (n & 1)) * 256;
      xs[half * 128 + row] = l0 + l1;
      if (n >= 2 && half == 0) wwait(bars + L::kOEmpty + o, ((n - 2) >> 1) & 1);
      if (bar_red_or(1, 256, aborted)) break;
      if (half == 0) {
        const float lsum = xs[row] + xs[128 + row];
        inv_l[o * 128 + row] = lsum > 0.f ? 1.f / lsum : 0.f;
        if (p.lse) {
          // natural-log log-sum-exp of the row: reference max plus log2 of
          // the sum (both in log2 units) times ln 2; -inf with no key
          // selected, 0 on padding rows
          const float v = row >= x.q_len ? 0.f
                          : (lsum > 0.f ? (m + __log2f(lsum)) * 0.69314718055994531f : -INFINITY);
          p.lse[x.group * p.lse_seq + 128LL * x.a + row] = v;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bars + L::kLFull + o);
    }
  } else {
    regs_dec<kRegsEpilogue>();
    // ===================== epilogue: one thread per query row =====================
    const int wq = warp - 12;
    const int row = wq * 32 + lane;
    const uint32_t t_lane = tmem_base + (uint32_t(wq * 32) << 16);
    uint32_t n = 0;
    for (long long it = it0; it < n_items; it += it_step, ++n) {
      const Item x = load_item(p, it);
      const int o = (int)(n & 1);
      if (!warp_wait(bars + L::kOFull + o, (n >> 1) & 1, abort_flag, p.status)) break;
      if (!warp_wait(bars + L::kLFull + o, (n >> 1) & 1, abort_flag, p.status)) break;
      tc_fence_after_sync();
      const float il = inv_l[o * 128 + row];
      const long long s = 128LL * x.a + row;
      __nv_bfloat16* orow = p.out + x.b * p.out_st.b + x.h * p.out_st.h + s * p.out_st.s;
      const __nv_bfloat16* grow =
          GATED ? p.gate + x.b * p.gate_st.b + x.h * p.gate_st.h + s * p.gate_st.s : nullptr;
      const float* oc = COMBINE ? p.out_c + (x.group * p.nq + x.ab) * (long long)D : nullptr;
      const bool real = row < x.q_len;
#pragma unroll
      for (int q0 = 0; q0 < D; q0 += 32) {
        uint32_t ov[32];
        if (x.num > 0) {
          VSA_TMEM_LD16(t_lane + kTmemO + D * o + q0, ov, 0);
          VSA_TMEM_LD16(t_lane + kTmemO + D * o + q0 + 16u, ov, 16);
          asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
        } else {
#pragma unroll
          for (int q = 0; q < 32; ++q) ov[q] = 0u;
        }
        if (real) {
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            float v[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) v[q] = __uint_as_float(ov[e + q]) * il;
            if (COMBINE) {
              const float4 c0 = *reinterpret_cast<const float4*>(oc + q0 + e);
              const float4 c1 = *reinterpret_cast<const float4*>(oc + q0 + e + 4);
              const float cv[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
              if (GATED) {
                const uint4 graw = *reinterpret_cast<const uint4*>(grow + q0 + e);
                const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&graw);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                  const float2 gf = __bfloat1622float2(g2[q]);
                  v[2 * q] = fmaf(cv[2 * q], gf.x, v[2 * q]);
                  v[2 * q + 1] = fmaf(cv[2 * q + 1], gf.y, v[2 * q + 1]);
                }
              } else {
#pragma unroll
                for (int q = 0; q < 8; ++q) v[q] += cv[q];
              }
            }
            *reinterpret_cast<uint4*>(orow + q0 + e) =
                make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                           pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
          }
        } else {
#pragma unroll
          for (int e = 0; e < 32; e += 8)
            *reinterpret_cast<uint4*>(orow + q0 + e) = make_uint4(0u, 0u, 0u, 0u);
        }
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(bars + L::kOEmpty + o);
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
// Self-test of the two products on operands staged by plain loads:
// mode 2: c[128][128] = a[128][D] . b[128][D]^T; mode 3: c[128][D] =
// a[128][128] . b[128][D] with a staged in TMEM as bf16.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(128, 1)
    selftest128_kernel(int mode, const __nv_bfloat16* a, const __nv_bfloat16* bm, float* cm) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint8_t* opa = smem;               // 32 KB
  uint8_t* opb = smem + 32768;       // 32 KB
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + 65536);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + 65536 + 8);
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const uint16_t* a16 = reinterpret_cast<const uint16_t*>(a);
  const uint16_t* b16 = reinterpret_cast<const uint16_t*>(bm);
  auto sw = [](uint32_t r, uint32_t chunk) { return r * 128u + ((chunk ^ (r & 7u)) << 4); };
  if (mode == 2) {
    for (int e = tid; e < 128 * D; e += 128) {
      const int r = e / D, col = e % D, dh = col / 64, cc = col % 64;
      *reinterpret_cast<uint16_t*>(opa + dh * 16384 + sw(r, cc / 8) + (cc % 8) * 2) = a16[e];
      *reinterpret_cast<uint16_t*>(opb + dh * 16384 + sw(r, cc / 8) + (cc % 8) * 2) = b16[e];
    }
  } else {
    for (int e = tid; e < 128 * D; e += 128) {
      const int r = e / D, col = e % D, dh = col / 64, cc = col % 64;
      *reinterpret_cast<uint16_t*>(opb + dh * 16384 + sw(r, cc / 8) + (cc % 8) * 2) = b16[e];
    }
  }
  fence_proxy_async_smem();
  if (tid == 0) {
    mbar_init(bar, 1);
    mbar_fence_init();
  }
  if (warp == 0) tmem_alloc(tmem_slot, 256);
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t t_lane = tmem_base + (uint32_t(warp * 32) << 16);
  if (mode == 3) {
    // row tid of a (128 bf16) -> 64 packed columns at column 128
    uint32_t pk[64];
    const int r = warp * 32 + lane;
    for (int q = 0; q < 64; ++q)
      pk[q] = (uint32_t)a16[r * 128 + 2 * q] | ((uint32_t)a16[r * 128 + 2 * q + 1] << 16);
#pragma unroll
    for (int q = 0; q < 4; ++q) VSA_TMEM_ST16(t_lane + 128u + 16u * q, pk, 16 * q);
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
    tc_fence_before_sync();
  }
  __syncthreads();
  tc_fence_after_sync();
  if (tid == 0) {
    if (mode == 2) issue_s<D>(tmem_base, sbase, sbase + 32768);
    else issue_pv<D>(tmem_base, tmem_base + 128u, sbase + 32768, false);
    umma_commit(bar);
  }
  int dummy_abort = 0;
  mbar_wait(bar, 0, &dummy_abort, nullptr);
  tc_fence_after_sync();
  const int cols = mode == 2 ? 128 : D;
  const int r = warp * 32 + lane;
  for (int q0 = 0; q0 < cols; q0 += 16) {
    uint32_t o[16];
    VSA_TMEM_LD16(t_lane + q0, o, 0);
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
    for (int q = 0; q < 16; ++q) cm[r * cols + q0 + q] = __uint_as_float(o[q]);
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, 256);
  }
}

}  // namespace b128

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
template <int D, bool COMBINE, bool GATED>
static int launch128_t(const SparseParams& p, const CUtensorMap& mq, const CUtensorMap& mk,
                       const CUtensorMap& mv, cudaStream_t stream) {
  using L = b128::Layout<D>;
  auto kern = b128::sparse128_fwd_kernel<D, COMBINE, GATED>;
  // The warpgroup register split assumes kLaunchRegs per thread at launch.
  static int regs_ok = -1;
  if (regs_ok < 0) {
    cudaFuncAttributes attr;
    regs_ok = (cudaFuncGetAttributes(&attr, kern) == cudaSuccess &&
               attr.numRegs == (int)b128::kLaunchRegs) ? 1 : 0;
  }
  if (!regs_ok) return VSA_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::kAlloc) !=
      cudaSuccess)
    return VSA_ERR_CUDA;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long n_items = ((long long)p.B * p.H * p.nq) << p.sub;
  const long long grid = n_items < sms ? n_items : sms;
  kern<<<(unsigned)grid, b128::kThreads, L::kAlloc, stream>>>(mq, mk, mv, p);
  return cudaGetLastError() == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

int launch_sparse128(const SparseParams& p_in, const void* q, Strides3 q_st, long long q_seq,
                     const void* k, Strides3 k_st, const void* v, Strides3 v_st, long long kv_seq,
                     int D, bool combine, bool gated, cudaStream_t stream) {
  if (p_in.nq <= 0 || p_in.H <= 0 || p_in.B <= 0) return VSA_OK;
  if (p_in.q_tok || p_in.kv_tok || p_in.varlen) return VSA_ERR_UNSUPPORTED;
  if (p_in.sub < 0 || p_in.sub > 1) return VSA_ERR_UNSUPPORTED;
  if (q_seq + 128 > 0x7FFFFFFFLL || kv_seq + 128 > 0x7FFFFFFFLL) return VSA_ERR_UNSUPPORTED;
  SparseParams p = p_in;
  CUtensorMap mq, mk, mv;
  if (!make_view_map_rows(&mq, &p.q_ax, q, D, q_seq, p.H, p.B, q_st, 128) ||
      !make_view_map_rows(&mk, &p.k_ax, k, D, kv_seq, p.H, p.B, k_st, 128) ||
      !make_view_map_rows(&mv, &p.v_ax, v, D, kv_seq, p.H, p.B, v_st, 128))
    return VSA_ERR_CUDA;
  if (D == 128) {
    if (!combine) return launch128_t<128, false, false>(p, mq, mk, mv, stream);
    if (gated) return launch128_t<128, true, true>(p, mq, mk, mv, stream);
    return launch128_t<128, true, false>(p, mq, mk, mv, stream);
  }
  if (!combine) return launch128_t<64, false, false>(p, mq, mk, mv, stream);
  if (gated) return launch128_t<64, true, true>(p, mq, mk, mv, stream);
  return launch128_t<64, true, false>(p, mq, mk, mv, stream);
}

int launch_selftest128(int mode, int D, const void* a, const void* b, float* c,
                       cudaStream_t stream) {
  const int smem = 65536 + 64 + 1024;
  if (D == 128) {
    cudaFuncSetAttribute(b128::selftest128_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    b128::selftest128_kernel<128><<<1, 128, smem, stream>>>(
        mode, static_cast<const __nv_bfloat16*>(a), static_cast<const __nv_bfloat16*>(b), c);
  } else {
    cudaFuncSetAttribute(b128::selftest128_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    b128::selftest128_kernel<64><<<1, 128, smem, stream>>>(
        mode, static_cast<const __nv_bfloat16*>(a), static_cast<const __nv_bfloat16*>(b), c);
  }
  return cudaGetLastError() == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

}  // namespace vsa
