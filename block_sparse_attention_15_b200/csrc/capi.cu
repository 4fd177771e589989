// C ABI of libvsa.so: argument checks, workspace carving, host-side block
// metadata, and the launch sequence of every entry point declared in vsa.h.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <mutex>
#include <vector>

#include "vsa.h"
#include "vsa_launch.h"

namespace vsa {

// Device status word: kernels record the first error of a launch sequence.
__device__ int g_device_status = 0;

// Page-locked staging of the small host tables some entries copy to the
// device (varlen block tables, host block sizes): per device, a ring of
// slots, each reused only after the copy that last read it has completed
// (one event per slot).  The copies are then truly asynchronous, and the host
// runs ahead of the stream by up to kStageSlots calls before it waits.
namespace {
constexpr int kStageSlots = 8;
constexpr int kMaxDevices = 64;
struct StageRing {
  std::mutex mu;
  void* buf[kStageSlots] = {};
  size_t cap[kStageSlots] = {};
  cudaEvent_t ev[kStageSlots] = {};
  bool pending[kStageSlots] = {};
  int next = 0;
};
StageRing g_stage[kMaxDevices];
}  // namespace

int stage_copy_h2d(void* dst, const void* src, size_t bytes, cudaStream_t st) {
  if (bytes == 0) return VSA_OK;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return VSA_ERR_CUDA;
  StageRing& r = g_stage[dev];
  std::lock_guard<std::mutex> lock(r.mu);
  const int i = r.next;
  r.next = (i + 1) % kStageSlots;
  if (r.pending[i] && cudaEventSynchronize(r.ev[i]) != cudaSuccess) return VSA_ERR_CUDA;
  r.pending[i] = false;
  if (!r.ev[i] && cudaEventCreateWithFlags(&r.ev[i], cudaEventDisableTiming) != cudaSuccess)
    return VSA_ERR_CUDA;
  if (r.cap[i] < bytes) {
    if (r.buf[i]) cudaFreeHost(r.buf[i]);
    r.buf[i] = nullptr;
    r.cap[i] = 0;
    const size_t want = bytes < 16384 ? 16384 : bytes;
    if (cudaMallocHost(&r.buf[i], want) != cudaSuccess) return VSA_ERR_CUDA;
    r.cap[i] = want;
  }
  memcpy(r.buf[i], src, bytes);
  if (cudaMemcpyAsync(dst, r.buf[i], bytes, cudaMemcpyHostToDevice, st) != cudaSuccess ||
      cudaEventRecord(r.ev[i], st) != cudaSuccess)
    return VSA_ERR_CUDA;
  r.pending[i] = true;
  return VSA_OK;
}

// The address is looked up once per device and cached (under a lock, so
// concurrent first calls from several host threads are safe).  The cache
// assumes the device's context lives as long as the process: a
// cudaDeviceReset between calls is not supported.
int* device_status_ptr() {
  static std::mutex mu;
  static int* cached[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!cached[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_device_status) != cudaSuccess) return nullptr;
    cached[dev] = static_cast<int*>(ptr);
  }
  return cached[dev];
}

static inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

static inline bool aligned16(const void* p) {
  return (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

// Optional timing events recorded around the kernels of vsa_forward.
static cudaEvent_t g_prof_events[4] = {nullptr, nullptr, nullptr, nullptr};
static bool g_prof_on = false;

float resolve_scale(float scale, int D) {
  return scale > 0.f ? scale : 1.0f / sqrtf((float)D);
}

static Strides3 to_strides(const vsa_strides& s) { return Strides3{s.batch, s.head, s.seq}; }

Strides3 bhsd_strides(int H, long long S, int D) {
  return Strides3{(long long)H * S * D, S * D, (long long)D};
}

Strides3 gate_strides(int H, long long S, int D) {
  return Strides3{S * H * D, (long long)D, (long long)H * D};
}

// A view is usable when every stride of an axis longer than one is a
// positive multiple of 8 elements (16 bytes: TMA and 16-byte loads).
static bool strides_ok(const Strides3& st, int B, int H, long long S) {
  auto ok = [](long long stride, long long extent) {
    return extent <= 1 || (stride > 0 && stride % 8 == 0);
  };
  return ok(st.b, B) && ok(st.h, H) && ok(st.s, S);
}

static bool layout_ok(const vsa_layout& L, int B, int H, long long Sq, long long Skv, bool gated) {
  return strides_ok(to_strides(L.q), B, H, Sq) && strides_ok(to_strides(L.k), B, H, Skv) &&
         strides_ok(to_strides(L.v), B, H, Skv) && strides_ok(to_strides(L.out), B, H, Sq) &&
         (!gated || strides_ok(to_strides(L.gate), B, H, Sq));
}

static void fill_layout(int kind, int B, int H, int Sq, int Skv, int D, vsa_layout* L) {
  (void)B;
  auto set = [](vsa_strides& s, long long b, long long h, long long q) {
    s.batch = b; s.head = h; s.seq = q;
  };
  if (kind == VSA_LAYOUT_BSHD) {
    set(L->q, (long long)Sq * H * D, D, (long long)H * D);
    set(L->out, (long long)Sq * H * D, D, (long long)H * D);
    set(L->k, (long long)Skv * H * D, D, (long long)H * D);
    set(L->v, (long long)Skv * H * D, D, (long long)H * D);
  } else {
    set(L->q, (long long)H * Sq * D, (long long)Sq * D, D);
    set(L->out, (long long)H * Sq * D, (long long)Sq * D, D);
    set(L->k, (long long)H * Skv * D, (long long)Skv * D, D);
    set(L->v, (long long)H * Skv * D, (long long)Skv * D, D);
  }
  // the gate ("compress_attn_weight") is [B, Sq, H, D] memory in both
  set(L->gate, (long long)Sq * H * D, D, (long long)H * D);
}


int check_forward_args(const ForwardArgs& a) {
  if (!a.q || !a.k || !a.v || !a.out || !a.q2k_idx || !a.q2k_num) return VSA_ERR_INVALID_ARG;
  if (a.B <= 0 || a.H <= 0 || a.Sq_pad <= 0 || a.Skv_pad <= 0 || a.topk < 1 || !(a.scale == a.scale))
    return VSA_ERR_INVALID_ARG;
  if (a.D != 64 && a.D != 128) return VSA_ERR_UNSUPPORTED;
  if (a.block != 64 && a.block != 128 && a.block != 256) return VSA_ERR_UNSUPPORTED;
  if (a.Sq_pad % a.block || a.Skv_pad % a.block) return VSA_ERR_SHAPE;
  const int nq = a.Sq_pad / a.block, nkv = a.Skv_pad / a.block;
  if (nq > VSA_MAX_BLOCKS || nkv > VSA_MAX_BLOCKS) return VSA_ERR_UNSUPPORTED;
  const int k_eff = a.topk < nkv ? a.topk : nkv;
  if (a.idx_stride < k_eff) return VSA_ERR_SHAPE;
  if (!aligned16(a.q) || !aligned16(a.k) || !aligned16(a.v) || !aligned16(a.out) ||
      (a.gate && !aligned16(a.gate)) || (a.out_c && !aligned16(a.out_c)))
    return VSA_ERR_INVALID_ARG;
  if (!strides_ok(a.q_st, a.B, a.H, a.Sq_pad) || !strides_ok(a.k_st, a.B, a.H, a.Skv_pad) ||
      !strides_ok(a.v_st, a.B, a.H, a.Skv_pad) || !strides_ok(a.out_st, a.B, a.H, a.Sq_pad) ||
      (a.gate && !strides_ok(a.gate_st, a.B, a.H, a.Sq_pad)))
    return VSA_ERR_UNSUPPORTED;
  return VSA_OK;
}

// The three launches of the forward on checked arguments, with the scratch
// regions carved from `scratch` (vsa_forward_workspace_size bytes, 256-byte
// aligned) in the documented order.  Every region is written in full by the
// kernel that produces it before any kernel reads it.
int launch_forward(const ForwardArgs& a, void* scratch, bool profile, cudaStream_t st) {
  const int B = a.B, H = a.H, D = a.D;
  const int nq = a.Sq_pad / a.block, nkv = a.Skv_pad / a.block;
  // the logit bound lets both sparse kernels skip their running-max checks
  // where it proves them unneeded
  const bool bound = true;
  const int k_eff = a.topk < nkv ? a.topk : nkv;
  int* status = device_status_ptr();
  if (!status) return VSA_ERR_CUDA;
  const bool prof = profile && g_prof_on;

  const size_t g = (size_t)B * H * D * sizeof(float);
  char* ws = static_cast<char*>(scratch);
  float* qc = reinterpret_cast<float*>(ws);
  ws += align256(g * nq);
  float* kc = reinterpret_cast<float*>(ws);
  ws += align256(g * nkv);
  float* vc = reinterpret_cast<float*>(ws);
  ws += align256(g * nkv);
  float* oc = a.out_c ? a.out_c : reinterpret_cast<float*>(ws);
  ws += align256(g * nq);
  // block row norms and the per-query-block logit bound
  const size_t G = (size_t)B * H;
  float* qn = reinterpret_cast<float*>(ws);
  float* kn = qn + G * nq;
  float* qk_bound = kn + G * nkv;

  PoolParams pp;
  pp.q = static_cast<const __nv_bfloat16*>(a.q);
  pp.k = static_cast<const __nv_bfloat16*>(a.k);
  pp.v = static_cast<const __nv_bfloat16*>(a.v);
  pp.q_st = a.q_st;
  pp.k_st = a.k_st;
  pp.v_st = a.v_st;
  pp.q_bs = a.q_block_sizes;
  pp.kv_bs = a.kv_block_sizes;
  pp.groups = B * H;
  pp.H = H;
  pp.block = a.block;
  pp.nq = nq;
  pp.nkv = nkv;
  pp.qc = qc;
  pp.kc = kc;
  pp.vc = vc;
  pp.qn = bound ? qn : nullptr;
  pp.kn = bound ? kn : nullptr;
  pp.status = status;
  if (prof) cudaEventRecord(g_prof_events[0], st);
  int rc = launch_pool(pp, D, st);
  if (rc != VSA_OK) return rc;
  if (prof) cudaEventRecord(g_prof_events[1], st);

  const float sc = resolve_scale(a.scale, D);
  CoarseParams cp;
  cp.qc = qc;
  cp.kc = kc;
  cp.vc = vc;
  cp.groups = B * H;
  cp.nq = nq;
  cp.nkv = nkv;
  cp.scale = sc;
  cp.topk = k_eff;
  cp.idx_stride = a.idx_stride;
  cp.q2k_idx = a.q2k_idx;
  cp.q2k_num = a.q2k_num;
  cp.out_c = oc;
  cp.qn = qn;
  cp.kn = kn;
  cp.qk_bound = bound ? qk_bound : nullptr;
  cp.bound_scale = sc * kLog2e * (1.f + 0x1p-8f);
  cp.status = status;
  rc = launch_coarse_topk(cp, D, st);
  if (rc != VSA_OK) return rc;
  if (prof) cudaEventRecord(g_prof_events[2], st);

  SparseParams sp;
  memset(&sp, 0, sizeof(sp));
  sp.out = static_cast<__nv_bfloat16*>(a.out);
  sp.out_st = a.out_st;
  sp.gate = static_cast<const __nv_bfloat16*>(a.gate);
  sp.gate_st = a.gate_st;
  sp.out_c = oc;
  sp.q2k_idx = a.q2k_idx;
  sp.q2k_num = a.q2k_num;
  sp.idx_stride = a.idx_stride;
  sp.q_bs = a.q_block_sizes;
  sp.kv_bs = a.kv_block_sizes;
  sp.B = B;
  sp.H = H;
  sp.nq = nq;
  sp.nkv = nkv;
  sp.scale_log2 = sc * kLog2e;
  sp.qk_bound = bound ? qk_bound : nullptr;
  sp.varlen = 0;
  sp.sub = a.block == 256 ? 1 : 0;  // 256-slot blocks: two 128-row halves
  sp.status = status;
  rc = a.block != 64
           ? launch_sparse128(sp, a.q, a.q_st, a.Sq_pad, a.k, a.k_st, a.v, a.v_st, a.Skv_pad, D,
                              /*combine=*/true, /*gated=*/a.gate != nullptr, st)
           : launch_sparse(sp, a.q, a.q_st, a.Sq_pad, a.k, a.k_st, a.v, a.v_st, a.Skv_pad, D,
                           /*combine=*/true, /*gated=*/a.gate != nullptr, st);
  if (rc != VSA_OK) return rc;
  if (prof) cudaEventRecord(g_prof_events[3], st);
  return VSA_OK;
}

}  // namespace vsa

using namespace vsa;

extern "C" {

const char* vsa_status_string(int status) {
  switch (status) {
    case VSA_OK: return "ok";
    case VSA_ERR_INVALID_ARG: return "invalid argument";
    case VSA_ERR_SHAPE: return "inconsistent shape";
    case VSA_ERR_UNSUPPORTED: return "unsupported configuration";
    case VSA_ERR_CUDA: return "CUDA error";
    case VSA_ERR_DEVICE_TIMEOUT: return "device barrier wait timed out";
    case VSA_ERR_INDEX_RANGE: return "block index out of range";
    case VSA_ERR_WORKSPACE: return "workspace missing, too small or misaligned";
    case VSA_ERR_BLOCK_SIZE: return "block size outside [1, 64]";
    default: return "unknown status";
  }
}

int vsa_abi_version(void) { return (2 << 16) | 1; }

int vsa_get_device_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return VSA_ERR_CUDA;
  int value = 0;
  if (cudaMemcpyFromSymbol(&value, g_device_status, sizeof(int)) != cudaSuccess) return VSA_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)) != cudaSuccess) return VSA_ERR_CUDA;
  return value;
}

// ---------------------------------------------------------------------------
// vsa_forward
// ---------------------------------------------------------------------------
size_t vsa_forward_workspace_size(int B, int H, int n_q_blocks, int n_kv_blocks, int D) {
  if (B <= 0 || H <= 0 || n_q_blocks <= 0 || n_kv_blocks <= 0 || D <= 0) return 0;
  const size_t g = (size_t)B * H * D * sizeof(float);
  const size_t norms = (size_t)B * H * (2 * (size_t)n_q_blocks + n_kv_blocks) * sizeof(float);
  return align256(g * n_q_blocks) * 2 + align256(g * n_kv_blocks) * 2 + align256(norms);
}

int vsa_make_layout(int kind, int B, int H, int Sq_pad, int Skv_pad, int D, vsa_layout* layout) {
  if (!layout || (kind != VSA_LAYOUT_BHSD && kind != VSA_LAYOUT_BSHD)) return VSA_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || Sq_pad <= 0 || Skv_pad <= 0 || D <= 0) return VSA_ERR_INVALID_ARG;
  fill_layout(kind, B, H, Sq_pad, Skv_pad, D, layout);
  return VSA_OK;
}

int vsa_forward_strided(const void* q, const void* k, const void* v, const void* gate,
                        const vsa_layout* layout, const int32_t* q_block_sizes,
                        const int32_t* kv_block_sizes, int B, int H, int Sq_pad, int Skv_pad,
                        int D, int block_size, int topk, float scale, void* out, int32_t* q2k_idx,
                        int32_t* q2k_num, int idx_stride, float* out_c, void* workspace,
                        size_t workspace_bytes, void* stream) {
  if (!layout) return VSA_ERR_INVALID_ARG;
  ForwardArgs a;
  a.block = block_size;
  a.q = q; a.k = k; a.v = v; a.gate = gate;
  a.q_st = to_strides(layout->q); a.k_st = to_strides(layout->k); a.v_st = to_strides(layout->v);
  a.out_st = to_strides(layout->out); a.gate_st = to_strides(layout->gate);
  a.q_block_sizes = q_block_sizes; a.kv_block_sizes = kv_block_sizes;
  a.B = B; a.H = H; a.Sq_pad = Sq_pad; a.Skv_pad = Skv_pad; a.D = D; a.topk = topk;
  a.scale = scale; a.out = out; a.q2k_idx = q2k_idx; a.q2k_num = q2k_num;
  a.idx_stride = idx_stride; a.out_c = out_c;
  int rc = check_forward_args(a);
  if (rc != VSA_OK) return rc;
  const size_t need = vsa_forward_workspace_size(B, H, Sq_pad / block_size, Skv_pad / block_size, D);
  if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return VSA_ERR_WORKSPACE;
  return launch_forward(a, workspace, /*profile=*/true, static_cast<cudaStream_t>(stream));
}

int vsa_forward(const void* q, const void* k, const void* v, const void* gate,
                const int32_t* q_block_sizes, const int32_t* kv_block_sizes, int B, int H,
                int Sq_pad, int Skv_pad, int D, int topk, float scale, void* out,
                int32_t* q2k_idx, int32_t* q2k_num, int idx_stride, float* out_c,
                void* workspace, size_t workspace_bytes, void* stream) {
  if (B <= 0 || H <= 0 || Sq_pad <= 0 || Skv_pad <= 0 || D <= 0) return VSA_ERR_INVALID_ARG;
  vsa_layout L;
  fill_layout(VSA_LAYOUT_BHSD, B, H, Sq_pad, Skv_pad, D, &L);
  return vsa_forward_strided(q, k, v, gate, &L, q_block_sizes, kv_block_sizes, B, H, Sq_pad,
                             Skv_pad, D, 64, topk, scale, out, q2k_idx, q2k_num, idx_stride, out_c,
                             workspace, workspace_bytes, stream);
}

int vsa_forward_bshd(const void* q, const void* k, const void* v, const void* gate,
                     const int32_t* q_block_sizes, const int32_t* kv_block_sizes, int B, int H,
                     int Sq_pad, int Skv_pad, int D, int topk, float scale, void* out,
                     int32_t* q2k_idx, int32_t* q2k_num, int idx_stride, float* out_c,
                     void* workspace, size_t workspace_bytes, void* stream) {
  if (B <= 0 || H <= 0 || Sq_pad <= 0 || Skv_pad <= 0 || D <= 0) return VSA_ERR_INVALID_ARG;
  vsa_layout L;
  fill_layout(VSA_LAYOUT_BSHD, B, H, Sq_pad, Skv_pad, D, &L);
  return vsa_forward_strided(q, k, v, gate, &L, q_block_sizes, kv_block_sizes, B, H, Sq_pad,
                             Skv_pad, D, 64, topk, scale, out, q2k_idx, q2k_num, idx_stride, out_c,
                             workspace, workspace_bytes, stream);
}

// ---------------------------------------------------------------------------
// block_sparse_attn_from_indices
// ---------------------------------------------------------------------------
size_t block_sparse_attn_from_indices_workspace_size(int B, int H, int n_q_blocks,
                                                     int n_kv_blocks) {
  if (B <= 0 || H <= 0 || n_q_blocks <= 0 || n_kv_blocks <= 0) return 0;
  return align256(index_bound_bytes(B * H, n_q_blocks, n_kv_blocks));
}

// Shared by block_sparse_attn_from_indices and block_sparse_attn: checks,
// the optional logit-bound pass, then the sparse kernel.
static int sparse_from_indices(const void* q, const void* k, const void* v,
                               const int32_t* q2k_idx, const int32_t* q2k_num,
                               const int32_t* q_block_sizes, const int32_t* kv_block_sizes, int B,
                               int H, int Sq_pad, int Skv_pad, int D, int block, int idx_stride,
                               float scale, void* out, float* lse, const vsa_layout* layout,
                               void* workspace, size_t workspace_bytes, cudaStream_t st) {
  if (!q || !k || !v || !out || !q2k_idx || !q2k_num) return VSA_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || Sq_pad <= 0 || Skv_pad <= 0 || idx_stride < 1 || !(scale == scale))
    return VSA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return VSA_ERR_UNSUPPORTED;
  if (block != 64 && block != 128 && block != 256) return VSA_ERR_UNSUPPORTED;
  if (Sq_pad % block || Skv_pad % block) return VSA_ERR_SHAPE;
  const int nq = Sq_pad / block, nkv = Skv_pad / block;
  if (idx_stride > VSA_MAX_BLOCKS) return VSA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return VSA_ERR_INVALID_ARG;
  vsa_layout L;
  if (layout) L = *layout;
  else fill_layout(VSA_LAYOUT_BHSD, B, H, Sq_pad, Skv_pad, D, &L);
  if (!layout_ok(L, B, H, Sq_pad, Skv_pad, false)) return VSA_ERR_UNSUPPORTED;
  if (workspace) {
    const size_t need = block_sparse_attn_from_indices_workspace_size(B, H, nq, nkv);
    if (workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
      return VSA_ERR_WORKSPACE;
  }
  int* status = device_status_ptr();
  if (!status) return VSA_ERR_CUDA;
  const float sc = resolve_scale(scale, D);
  const float* qk_bound = nullptr;
  if (workspace) {
    // logit bound of every item from block row norms and its selection
    BoundParams bp;
    memset(&bp, 0, sizeof(bp));
    bp.q = static_cast<const __nv_bfloat16*>(q);
    bp.k = static_cast<const __nv_bfloat16*>(k);
    bp.q_st = to_strides(L.q);
    bp.k_st = to_strides(L.k);
    bp.q_seq = Sq_pad;
    bp.kv_seq = Skv_pad;
    bp.kv_len = kv_block_sizes;
    bp.q2k_idx = q2k_idx;
    bp.q2k_num = q2k_num;
    bp.idx_stride = idx_stride;
    bp.B = B;
    bp.H = H;
    bp.nqb = nq;
    bp.nkvb = nkv;
    bp.block = block;
    bp.bound_scale = sc * kLog2e * (1.f + 0x1p-8f);
    bp.qn = static_cast<float*>(workspace);
    bp.kn = bp.qn + (size_t)B * H * nq;
    bp.qk_bound = bp.kn + (size_t)B * H * nkv;
    int rc = launch_index_bound(bp, D, st);
    if (rc != VSA_OK) return rc;
    qk_bound = bp.qk_bound;
  }
  SparseParams sp;
  memset(&sp, 0, sizeof(sp));
  sp.out = static_cast<__nv_bfloat16*>(out);
  sp.out_st = to_strides(L.out);
  sp.q2k_idx = q2k_idx;
  sp.q2k_num = q2k_num;
  sp.idx_stride = idx_stride;
  sp.q_bs = q_block_sizes;
  sp.kv_bs = kv_block_sizes;
  sp.B = B;
  sp.H = H;
  sp.nq = nq;
  sp.nkv = nkv;
  sp.scale_log2 = sc * kLog2e;
  sp.qk_bound = qk_bound;
  sp.lse = lse;
  sp.lse_seq = Sq_pad;
  sp.status = status;
  sp.sub = block == 256 ? 1 : 0;
  if (block != 64)
    return launch_sparse128(sp, q, to_strides(L.q), Sq_pad, k, to_strides(L.k), v, to_strides(L.v),
                            Skv_pad, D, false, false, st);
  return launch_sparse(sp, q, to_strides(L.q), Sq_pad, k, to_strides(L.k), v, to_strides(L.v),
                       Skv_pad, D, false, false, st);
}

int block_sparse_attn_from_indices(const void* q, const void* k, const void* v,
                                   const int32_t* q2k_idx, const int32_t* q2k_num,
                                   const int32_t* q_block_sizes, const int32_t* kv_block_sizes,
                                   int B, int H, int Sq_pad, int Skv_pad, int D, int block_size,
                                   int idx_stride, float scale, void* out, float* lse,
                                   const vsa_layout* layout, void* workspace,
                                   size_t workspace_bytes, void* stream) {
  return sparse_from_indices(q, k, v, q2k_idx, q2k_num, q_block_sizes, kv_block_sizes, B, H,
                             Sq_pad, Skv_pad, D, block_size, idx_stride, scale, out, lse, layout,
                             workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
}

// ---------------------------------------------------------------------------
// block_sparse_attn (bool block map)
// ---------------------------------------------------------------------------
int block_sparse_attn(const void* q, const void* k, const void* v, const uint8_t* block_map,
                      const int32_t* q_block_sizes, const int32_t* kv_block_sizes, int B, int H,
                      int Sq_pad, int Skv_pad, int D, int block_size, float scale, void* out,
                      int32_t* q2k_idx, int32_t* q2k_num, const vsa_layout* layout,
                      void* workspace, size_t workspace_bytes, void* stream) {
  if (!block_map || !q2k_idx || !q2k_num) return VSA_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || Sq_pad <= 0 || Skv_pad <= 0) return VSA_ERR_INVALID_ARG;
  if (block_size != 64 && block_size != 128 && block_size != 256) return VSA_ERR_UNSUPPORTED;
  if (Sq_pad % block_size || Skv_pad % block_size) return VSA_ERR_SHAPE;
  const int nq = Sq_pad / block_size, nkv = Skv_pad / block_size;
  if (nkv > VSA_MAX_BLOCKS) return VSA_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int rc = launch_mask_to_indices(block_map, (long long)B * H * nq, nkv, q2k_idx, q2k_num, st);
  if (rc != VSA_OK) return rc;
  return sparse_from_indices(q, k, v, q2k_idx, q2k_num, q_block_sizes, kv_block_sizes, B, H,
                             Sq_pad, Skv_pad, D, block_size, nkv, scale, out, nullptr, layout,
                             workspace, workspace_bytes, st);
}

// ---------------------------------------------------------------------------
// block_sparse_attn_varlen
// ---------------------------------------------------------------------------
size_t block_sparse_attn_varlen_workspace_size(int n_seqs, int total_q_blocks,
                                               int total_kv_blocks, int H) {
  if (n_seqs <= 0 || total_q_blocks <= 0 || total_kv_blocks <= 0 || H <= 0) return 0;
  // block tables, then block row norms and the per-query-block logit bound
  return align256(sizeof(int32_t) * (4 * (size_t)total_q_blocks + 2 * (size_t)total_kv_blocks)) +
         align256(sizeof(float) * (size_t)H * (2 * (size_t)total_q_blocks + total_kv_blocks));
}

// Resolve one side's blocks: per block first token row and size.
static int resolve_blocks(const int32_t* cu, const int32_t* sizes, const int32_t* cu_blocks,
                          int n, std::vector<int32_t>& tok, std::vector<int32_t>& len,
                          std::vector<int32_t>& first_block) {
  first_block.assign(n + 1, 0);
  if (cu[0] != 0) return VSA_ERR_SHAPE;
  for (int i = 0; i < n; ++i) {
    const long long L = (long long)cu[i + 1] - cu[i];
    if (L <= 0) return VSA_ERR_SHAPE;  // zero-token sequences are rejected
    if (sizes) {
      if (!cu_blocks) return VSA_ERR_INVALID_ARG;
      if (cu_blocks[0] != 0 || cu_blocks[i + 1] <= cu_blocks[i]) return VSA_ERR_SHAPE;
      long long t = cu[i];
      for (int j = cu_blocks[i]; j < cu_blocks[i + 1]; ++j) {
        const int s = sizes[j];
        if (s < 1 || s > 64) return VSA_ERR_BLOCK_SIZE;
        tok.push_back((int32_t)t);
        len.push_back(s);
        t += s;
      }
      if (t != cu[i + 1]) return VSA_ERR_SHAPE;  // block sizes must cover the sequence
    } else {
      for (long long t = cu[i]; t < cu[i + 1]; t += 64) {
        tok.push_back((int32_t)t);
        len.push_back((int32_t)((cu[i + 1] - t) < 64 ? (cu[i + 1] - t) : 64));
      }
    }
    first_block[i + 1] = (int32_t)tok.size();
  }
  return VSA_OK;
}

// Host-resolved varlen block tables: per packed query block its first token
// row, size, first KV block of its sequence and that sequence's KV block
// count; per packed KV block its first token row and size.
struct VarlenTables {
  std::vector<int32_t> table;  // qtok | qlen | kvbase | kvcount (nqb each), ktok | klen (nkvb each)
  int nqb = 0, nkvb = 0;
};

static int varlen_tables(const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_kv,
                         const int32_t* q_block_sizes, const int32_t* cu_q_blocks,
                         const int32_t* kv_block_sizes, const int32_t* cu_kv_blocks, int n_seqs,
                         VarlenTables& t) {
  std::vector<int32_t> qtok, qlen, qfirst, ktok, klen, kfirst;
  int rc = resolve_blocks(cu_seqlens_q, q_block_sizes, cu_q_blocks, n_seqs, qtok, qlen, qfirst);
  if (rc != VSA_OK) return rc;
  rc = resolve_blocks(cu_seqlens_kv, kv_block_sizes, cu_kv_blocks, n_seqs, ktok, klen, kfirst);
  if (rc != VSA_OK) return rc;
  const int nqb = (int)qtok.size(), nkvb = (int)ktok.size();
  t.nqb = nqb;
  t.nkvb = nkvb;
  t.table.assign(4 * (size_t)nqb + 2 * (size_t)nkvb, 0);
  int32_t* t_qtok = t.table.data();
  int32_t* t_qlen = t_qtok + nqb;
  int32_t* t_kvbase = t_qlen + nqb;
  int32_t* t_kvcount = t_kvbase + nqb;
  int32_t* t_ktok = t_kvcount + nqb;
  int32_t* t_klen = t_ktok + nkvb;
  for (int i = 0; i < n_seqs; ++i) {
    for (int a = qfirst[i]; a < qfirst[i + 1]; ++a) {
      t_qtok[a] = qtok[a];
      t_qlen[a] = qlen[a];
      t_kvbase[a] = kfirst[i];
      t_kvcount[a] = kfirst[i + 1] - kfirst[i];
    }
  }
  memcpy(t_ktok, ktok.data(), sizeof(int32_t) * nkvb);
  memcpy(t_klen, klen.data(), sizeof(int32_t) * nkvb);
  return VSA_OK;
}

int block_sparse_attn_varlen(const void* q, const void* k, const void* v,
                             const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_kv,
                             const int32_t* q_block_sizes, const int32_t* cu_q_blocks,
                             const int32_t* kv_block_sizes, const int32_t* cu_kv_blocks,
                             int n_seqs, int H, int D, const int32_t* q2k_idx,
                             const int32_t* q2k_num, int idx_stride, float scale, void* out,
                             float* lse, int64_t* pack_index_q, int64_t* pack_index_kv,
                             int32_t* q2k_idx_rebased, void* workspace, size_t workspace_bytes,
                             void* stream) {
  if (!q || !k || !v || !out || !q2k_idx || !q2k_num || !cu_seqlens_q || !cu_seqlens_kv)
    return VSA_ERR_INVALID_ARG;
  if (n_seqs <= 0) return VSA_ERR_SHAPE;  // empty batch
  if (H <= 0 || idx_stride < 1 || !(scale == scale)) return VSA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return VSA_ERR_UNSUPPORTED;
  if (idx_stride > VSA_MAX_BLOCKS) return VSA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return VSA_ERR_INVALID_ARG;
  VarlenTables vt;
  int rc = varlen_tables(cu_seqlens_q, cu_seqlens_kv, q_block_sizes, cu_q_blocks, kv_block_sizes,
                         cu_kv_blocks, n_seqs, vt);
  if (rc != VSA_OK) return rc;
  const int nqb = vt.nqb, nkvb = vt.nkvb;
  const std::vector<int32_t>& table = vt.table;
  const size_t need = block_sparse_attn_varlen_workspace_size(n_seqs, nqb, nkvb, H);
  if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return VSA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t* dtab = static_cast<int32_t*>(workspace);
  // through the page-locked ring, so `table` may be released right after
  if ((rc = stage_copy_h2d(dtab, table.data(), sizeof(int32_t) * table.size(), st)) != VSA_OK)
    return rc;
  int* status = device_status_ptr();
  if (!status) return VSA_ERR_CUDA;
  const int32_t* d_qtok = dtab;
  const int32_t* d_qlen = d_qtok + nqb;
  const int32_t* d_kvbase = d_qlen + nqb;
  const int32_t* d_kvcount = d_kvbase + nqb;
  const int32_t* d_ktok = d_kvcount + nqb;
  const int32_t* d_klen = d_ktok + nkvb;
  if (pack_index_q && (rc = launch_varlen_aux(d_qtok, d_qlen, nqb, pack_index_q, st)) != VSA_OK)
    return rc;
  if (pack_index_kv && (rc = launch_varlen_aux(d_ktok, d_klen, nkvb, pack_index_kv, st)) != VSA_OK)
    return rc;
  if (q2k_idx_rebased &&
      (rc = launch_rebase(q2k_idx, q2k_num, d_kvbase, d_kvcount, H, nqb, idx_stride,
                          q2k_idx_rebased, status, st)) != VSA_OK)
    return rc;
  const long long total_q = cu_seqlens_q[n_seqs], total_kv = cu_seqlens_kv[n_seqs];
  const float sc = resolve_scale(scale, D);
  // logit bound (lets the sparse kernel skip its running-max check where it
  // proves the check unneeded): block row norms, then per query block over
  // the blocks it selected
  float* qn = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                       align256(sizeof(int32_t) * table.size()));
  // token-packed [H, total, D] tensors as [1, H, total, D] views
  const Strides3 q_st{0, total_q * D, D}, kv_st{0, total_kv * D, D};
  BoundParams bp;
  memset(&bp, 0, sizeof(bp));
  bp.q = static_cast<const __nv_bfloat16*>(q);
  bp.k = static_cast<const __nv_bfloat16*>(k);
  bp.q_st = q_st;
  bp.k_st = kv_st;
  bp.q_seq = total_q;
  bp.kv_seq = total_kv;
  bp.q_tok = d_qtok;
  bp.kv_tok = d_ktok;
  bp.kv_len = d_klen;
  bp.q_kv_base = d_kvbase;
  bp.q_kv_count = d_kvcount;
  bp.q2k_idx = q2k_idx;
  bp.q2k_num = q2k_num;
  bp.idx_stride = idx_stride;
  bp.B = 1;
  bp.H = H;
  bp.nqb = nqb;
  bp.nkvb = nkvb;
  bp.bound_scale = sc * kLog2e * (1.f + 0x1p-8f);
  bp.qn = qn;
  bp.kn = qn + (size_t)H * nqb;
  bp.qk_bound = bp.kn + (size_t)H * nkvb;
  if ((rc = launch_index_bound(bp, D, st)) != VSA_OK) return rc;
  SparseParams sp;
  memset(&sp, 0, sizeof(sp));
  sp.out = static_cast<__nv_bfloat16*>(out);
  sp.out_st = q_st;
  sp.q2k_idx = q2k_idx;
  sp.q2k_num = q2k_num;
  sp.idx_stride = idx_stride;
  sp.q_bs = d_qlen;
  sp.kv_bs = d_klen;
  sp.q_tok = d_qtok;
  sp.kv_tok = d_ktok;
  sp.q_kv_base = d_kvbase;
  sp.q_kv_count = d_kvcount;
  sp.B = 1;
  sp.H = H;
  sp.nq = nqb;
  sp.nkv = nkvb;
  sp.scale_log2 = sc * kLog2e;
  sp.qk_bound = bp.qk_bound;
  sp.lse = lse;
  sp.lse_seq = total_q;
  sp.varlen = 1;
  sp.status = status;
  return launch_sparse(sp, q, q_st, total_q, k, kv_st, v, kv_st, total_kv, D, false, false, st);
}

// ---------------------------------------------------------------------------
// backward of block_sparse_attn_from_indices and of the varlen entry
// ---------------------------------------------------------------------------
static size_t bwd_scratch_bytes(long long groups, long long q_rows_per_group, int nqb, int nkvb) {
  return align256(sizeof(float) * (size_t)(groups * q_rows_per_group)) +
         align256(sizeof(int32_t) * (size_t)groups * nkvb * nqb) +
         align256(sizeof(int32_t) * (size_t)groups * nkvb);
}

size_t block_sparse_attn_backward_workspace_size(int B, int H, int Sq_pad, int n_kv_blocks) {
  if (B <= 0 || H <= 0 || Sq_pad <= 0 || Sq_pad % 64 || n_kv_blocks <= 0) return 0;
  return bwd_scratch_bytes((long long)B * H, Sq_pad, Sq_pad / 64, n_kv_blocks);
}

static void carve_bwd(BwdParams& bp, void* workspace, long long groups, long long q_rows, int nqb,
                      int nkvb) {
  char* ws = static_cast<char*>(workspace);
  bp.delta = reinterpret_cast<float*>(ws);
  ws += align256(sizeof(float) * (size_t)(groups * q_rows));
  bp.k2q = reinterpret_cast<int32_t*>(ws);
  ws += align256(sizeof(int32_t) * (size_t)groups * nkvb * nqb);
  bp.k2q_num = reinterpret_cast<int32_t*>(ws);
}

// The 64-slot backward on checked arguments; `workspace` holds at least
// block_sparse_attn_backward_workspace_size(B, H, Sq_pad, Skv_pad / 64) bytes.
static int backward64(const void* q, const void* k, const void* v, const void* out,
                      const void* dout, const float* lse, const int32_t* q2k_idx,
                      const int32_t* q2k_num, const int32_t* q_block_sizes,
                      const int32_t* kv_block_sizes, int B, int H, int Sq_pad, int Skv_pad, int D,
                      int idx_stride, float scale, void* dq, void* dk, void* dv, void* workspace,
                      int* status, cudaStream_t st) {
  const int nq = Sq_pad / 64, nkv = Skv_pad / 64;
  const float sc = resolve_scale(scale, D);
  BwdParams bp;
  memset(&bp, 0, sizeof(bp));
  bp.q = static_cast<const __nv_bfloat16*>(q);
  bp.k = static_cast<const __nv_bfloat16*>(k);
  bp.v = static_cast<const __nv_bfloat16*>(v);
  bp.dout = static_cast<const __nv_bfloat16*>(dout);
  bp.q_st = bp.do_st = bp.dq_st = bhsd_strides(H, Sq_pad, D);
  bp.k_st = bp.v_st = bp.dk_st = bp.dv_st = bhsd_strides(H, Skv_pad, D);
  bp.lse = lse;
  bp.q_seq = Sq_pad;
  bp.kv_seq = Skv_pad;
  bp.q2k_idx = q2k_idx;
  bp.q2k_num = q2k_num;
  bp.idx_stride = idx_stride;
  bp.q_bs = q_block_sizes;
  bp.kv_bs = kv_block_sizes;
  bp.dq = static_cast<__nv_bfloat16*>(dq);
  bp.dk = static_cast<__nv_bfloat16*>(dk);
  bp.dv = static_cast<__nv_bfloat16*>(dv);
  bp.B = B;
  bp.H = H;
  bp.nq = nq;
  bp.nkv = nkv;
  bp.scale = sc;
  bp.scale_log2 = sc * kLog2e;
  bp.status = status;
  carve_bwd(bp, workspace, (long long)B * H, Sq_pad, nq, nkv);
  return launch_backward(bp, out, bhsd_strides(H, Sq_pad, D), D, st);
}

// Argument checks shared by both backward entries.  The limits apply to the
// 64-slot selection the passes run on: Sq_pad / 64 and Skv_pad / 64 blocks,
// index rows idx_stride * block / 64 wide.
static int check_backward_args(const void* q, const void* k, const void* v, const void* out,
                               const void* dout, const float* lse, const int32_t* q2k_idx,
                               const int32_t* q2k_num, void* dq, void* dk, void* dv, int B, int H,
                               int Sq_pad, int Skv_pad, int D, int block, int idx_stride,
                               float scale) {
  if (!q || !k || !v || !out || !dout || !lse || !q2k_idx || !q2k_num || !dq || !dk || !dv)
    return VSA_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || Sq_pad <= 0 || Skv_pad <= 0 || idx_stride < 1 || !(scale == scale))
    return VSA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return VSA_ERR_UNSUPPORTED;
  if (block != 64 && block != 128 && block != 256) return VSA_ERR_UNSUPPORTED;
  if (Sq_pad % block || Skv_pad % block) return VSA_ERR_SHAPE;
  const long long stride64 = (long long)idx_stride * (block / 64);
  if (stride64 > VSA_MAX_BLOCKS || Sq_pad / 64 > VSA_MAX_BLOCKS || Skv_pad / 64 > VSA_MAX_BLOCKS)
    return VSA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(dout) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return VSA_ERR_INVALID_ARG;
  return VSA_OK;
}

int block_sparse_attn_backward(const void* q, const void* k, const void* v, const void* out,
                               const void* dout, const float* lse, const int32_t* q2k_idx,
                               const int32_t* q2k_num, const int32_t* q_block_sizes,
                               const int32_t* kv_block_sizes, int B, int H, int Sq_pad,
                               int Skv_pad, int D, int idx_stride, float scale, void* dq,
                               void* dk, void* dv, void* workspace, size_t workspace_bytes,
                               void* stream) {
  int rc = check_backward_args(q, k, v, out, dout, lse, q2k_idx, q2k_num, dq, dk, dv, B, H, Sq_pad,
                               Skv_pad, D, 64, idx_stride, scale);
  if (rc != VSA_OK) return rc;
  const size_t need = block_sparse_attn_backward_workspace_size(B, H, Sq_pad, Skv_pad / 64);
  if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return VSA_ERR_WORKSPACE;
  int* status = device_status_ptr();
  if (!status) return VSA_ERR_CUDA;
  return backward64(q, k, v, out, dout, lse, q2k_idx, q2k_num, q_block_sizes, kv_block_sizes, B, H,
                    Sq_pad, Skv_pad, D, idx_stride, scale, dq, dk, dv, workspace, status,
                    static_cast<cudaStream_t>(stream));
}

// Bytes of the 64-slot copy of a block-128/256 selection: index rows,
// counts, query and key sub-block sizes.
static size_t expand_bytes(long long groups, int nq, int nkv, int idx_stride, int shift) {
  const size_t nq64 = (size_t)nq << shift, nkv64 = (size_t)nkv << shift;
  return align256(sizeof(int32_t) * (size_t)groups * nq64 * ((size_t)idx_stride << shift)) +
         align256(sizeof(int32_t) * (size_t)groups * nq64) + align256(sizeof(int32_t) * nq64) +
         align256(sizeof(int32_t) * nkv64);
}

static int block_shift(int block) { return block == 256 ? 2 : (block == 128 ? 1 : 0); }

size_t block_sparse_attn_backward_ex_workspace_size(int B, int H, int Sq_pad, int Skv_pad,
                                                    int block_size, int idx_stride) {
  if (B <= 0 || H <= 0 || Sq_pad <= 0 || Skv_pad <= 0 || idx_stride < 1) return 0;
  if (block_size != 64 && block_size != 128 && block_size != 256) return 0;
  if (Sq_pad % block_size || Skv_pad % block_size) return 0;
  const int shift = block_shift(block_size);
  const size_t base = block_sparse_attn_backward_workspace_size(B, H, Sq_pad, Skv_pad / 64);
  if (!shift) return base;
  return base + expand_bytes((long long)B * H, Sq_pad / block_size, Skv_pad / block_size,
                             idx_stride, shift);
}

int block_sparse_attn_backward_ex(const void* q, const void* k, const void* v, const void* out,
                                  const void* dout, const float* lse, const int32_t* q2k_idx,
                                  const int32_t* q2k_num, const int32_t* q_block_sizes,
                                  const int32_t* kv_block_sizes, int B, int H, int Sq_pad,
                                  int Skv_pad, int D, int block_size, int idx_stride, float scale,
                                  void* dq, void* dk, void* dv, void* workspace,
                                  size_t workspace_bytes, void* stream) {
  int rc = check_backward_args(q, k, v, out, dout, lse, q2k_idx, q2k_num, dq, dk, dv, B, H, Sq_pad,
                               Skv_pad, D, block_size, idx_stride, scale);
  if (rc != VSA_OK) return rc;
  const size_t need =
      block_sparse_attn_backward_ex_workspace_size(B, H, Sq_pad, Skv_pad, block_size, idx_stride);
  if (!workspace || !need || workspace_bytes < need ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return VSA_ERR_WORKSPACE;
  int* status = device_status_ptr();
  if (!status) return VSA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int shift = block_shift(block_size);
  if (!shift)
    return backward64(q, k, v, out, dout, lse, q2k_idx, q2k_num, q_block_sizes, kv_block_sizes, B,
                      H, Sq_pad, Skv_pad, D, idx_stride, scale, dq, dk, dv, workspace, status, st);
  // the selection over 64-slot sub-blocks, after the 64-slot scratch
  ExpandParams e;
  memset(&e, 0, sizeof(e));
  e.q2k_idx = q2k_idx;
  e.q2k_num = q2k_num;
  e.q_bs = q_block_sizes;
  e.kv_bs = kv_block_sizes;
  e.groups = (long long)B * H;
  e.nq = Sq_pad / block_size;
  e.nkv = Skv_pad / block_size;
  e.idx_stride = idx_stride;
  e.shift = shift;
  e.status = status;
  char* ws = static_cast<char*>(workspace) +
             block_sparse_attn_backward_workspace_size(B, H, Sq_pad, Skv_pad / 64);
  const size_t nq64 = (size_t)e.nq << shift;
  e.idx64 = reinterpret_cast<int32_t*>(ws);
  ws += align256(sizeof(int32_t) * (size_t)e.groups * nq64 * ((size_t)idx_stride << shift));
  e.num64 = reinterpret_cast<int32_t*>(ws);
  ws += align256(sizeof(int32_t) * (size_t)e.groups * nq64);
  e.q_bs64 = reinterpret_cast<int32_t*>(ws);
  ws += align256(sizeof(int32_t) * nq64);
  e.kv_bs64 = reinterpret_cast<int32_t*>(ws);
  rc = launch_expand_selection(e, st);
  if (rc != VSA_OK) return rc;
  return backward64(q, k, v, out, dout, lse, e.idx64, e.num64, e.q_bs64, e.kv_bs64, B, H, Sq_pad,
                    Skv_pad, D, idx_stride << shift, scale, dq, dk, dv, workspace, status, st);
}

size_t block_sparse_attn_varlen_backward_workspace_size(int n_seqs, int total_q_blocks,
                                                        int total_kv_blocks, int H, int total_q) {
  if (n_seqs <= 0 || total_q_blocks <= 0 || total_kv_blocks <= 0 || H <= 0 || total_q <= 0) return 0;
  return align256(sizeof(int32_t) * (4 * (size_t)total_q_blocks + 2 * (size_t)total_kv_blocks)) +
         bwd_scratch_bytes(H, total_q, total_q_blocks, total_kv_blocks);
}

int block_sparse_attn_varlen_backward(
    const void* q, const void* k, const void* v, const void* out, const void* dout, const float* lse,
    const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_kv, const int32_t* q_block_sizes,
    const int32_t* cu_q_blocks, const int32_t* kv_block_sizes, const int32_t* cu_kv_blocks,
    int n_seqs, int H, int D, const int32_t* q2k_idx, const int32_t* q2k_num, int idx_stride,
    float scale, void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes,
    void* stream) {
  if (!q || !k || !v || !out || !dout || !lse || !q2k_idx || !q2k_num || !dq || !dk || !dv ||
      !cu_seqlens_q || !cu_seqlens_kv)
    return VSA_ERR_INVALID_ARG;
  if (n_seqs <= 0) return VSA_ERR_SHAPE;
  if (H <= 0 || idx_stride < 1 || !(scale == scale)) return VSA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return VSA_ERR_UNSUPPORTED;
  if (idx_stride > VSA_MAX_BLOCKS) return VSA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(dout) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return VSA_ERR_INVALID_ARG;
  VarlenTables vt;
  int rc = varlen_tables(cu_seqlens_q, cu_seqlens_kv, q_block_sizes, cu_q_blocks, kv_block_sizes,
                         cu_kv_blocks, n_seqs, vt);
  if (rc != VSA_OK) return rc;
  const int nqb = vt.nqb, nkvb = vt.nkvb;
  if (nqb > 0xFFFF) return VSA_ERR_UNSUPPORTED;  // k2q packs query block numbers in 16 bits
  const long long total_q = cu_seqlens_q[n_seqs], total_kv = cu_seqlens_kv[n_seqs];
  const size_t need = block_sparse_attn_varlen_backward_workspace_size(n_seqs, nqb, nkvb, H, (int)total_q);
  if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return VSA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t* dtab = static_cast<int32_t*>(workspace);
  if ((rc = stage_copy_h2d(dtab, vt.table.data(), sizeof(int32_t) * vt.table.size(), st)) != VSA_OK)
    return rc;
  int* status = device_status_ptr();
  if (!status) return VSA_ERR_CUDA;
  const float sc = resolve_scale(scale, D);
  const Strides3 q_st{0, total_q * D, D}, kv_st{0, total_kv * D, D};
  BwdParams bp;
  memset(&bp, 0, sizeof(bp));
  bp.q = static_cast<const __nv_bfloat16*>(q);
  bp.k = static_cast<const __nv_bfloat16*>(k);
  bp.v = static_cast<const __nv_bfloat16*>(v);
  bp.dout = static_cast<const __nv_bfloat16*>(dout);
  bp.q_st = bp.do_st = bp.dq_st = q_st;
  bp.k_st = bp.v_st = bp.dk_st = bp.dv_st = kv_st;
  bp.lse = lse;
  bp.q_seq = total_q;
  bp.kv_seq = total_kv;
  bp.q2k_idx = q2k_idx;
  bp.q2k_num = q2k_num;
  bp.idx_stride = idx_stride;
  bp.q_tok = dtab;
  bp.q_bs = dtab + nqb;
  bp.q_kv_base = dtab + 2 * nqb;
  bp.q_kv_count = dtab + 3 * nqb;
  bp.kv_tok = dtab + 4 * nqb;
  bp.kv_bs = dtab + 4 * nqb + nkvb;
  bp.dq = static_cast<__nv_bfloat16*>(dq);
  bp.dk = static_cast<__nv_bfloat16*>(dk);
  bp.dv = static_cast<__nv_bfloat16*>(dv);
  bp.B = 1;
  bp.H = H;
  bp.nq = nqb;
  bp.nkv = nkvb;
  bp.scale = sc;
  bp.scale_log2 = sc * kLog2e;
  bp.varlen = 1;
  bp.status = status;
  carve_bwd(bp, static_cast<char*>(workspace) + align256(sizeof(int32_t) * vt.table.size()), H,
            total_q, nqb, nkvb);
  return launch_backward(bp, out, q_st, D, st);
}

// ---------------------------------------------------------------------------
// build_vsa_metadata (host) and the device gather / scatter
// ---------------------------------------------------------------------------
int build_vsa_metadata(int T, int Hh, int W, int tT, int tH, int tW,
                       int64_t* tile_partition_indices, int64_t* reverse_tile_partition_indices,
                       int32_t* variable_block_sizes, int64_t* non_pad_index,
                       int64_t* slot_token, int32_t* n_tiles) {
  if (T <= 0 || Hh <= 0 || W <= 0 || tT <= 0 || tH <= 0 || tW <= 0) return VSA_ERR_INVALID_ARG;
  const int vol = tT * tH * tW;
  if (vol > 256) return VSA_ERR_INVALID_ARG;
  const int nT = (T + tT - 1) / tT, nH = (Hh + tH - 1) / tH, nW = (W + tW - 1) / tW;
  const long long ntiles = (long long)nT * nH * nW;
  if (ntiles > 0x7FFFFFFFLL) return VSA_ERR_UNSUPPORTED;
  if (n_tiles) *n_tiles = (int32_t)ntiles;
  long long pos = 0;
  long long tile = 0;
  for (int bt = 0; bt < nT; ++bt) {
    for (int bh = 0; bh < nH; ++bh) {
      for (int bw = 0; bw < nW; ++bw, ++tile) {
        int count = 0;
        const int t1 = (bt + 1) * tT < T ? (bt + 1) * tT : T;
        const int h1 = (bh + 1) * tH < Hh ? (bh + 1) * tH : Hh;
        const int w1 = (bw + 1) * tW < W ? (bw + 1) * tW : W;
        for (int t = bt * tT; t < t1; ++t) {
          for (int h = bh * tH; h < h1; ++h) {
            for (int w = bw * tW; w < w1; ++w) {
              const int64_t token = ((int64_t)t * Hh + h) * W + w;
              const int64_t slot = tile * vol + count;
              if (tile_partition_indices) tile_partition_indices[pos] = token;
              if (reverse_tile_partition_indices) reverse_tile_partition_indices[token] = pos;
              if (non_pad_index) non_pad_index[pos] = slot;
              if (slot_token) slot_token[slot] = token;
              ++pos;
              ++count;
            }
          }
        }
        if (variable_block_sizes) variable_block_sizes[tile] = count;
        if (slot_token) {
          for (int s = count; s < vol; ++s) slot_token[tile * vol + s] = -1;
        }
      }
    }
  }
  return VSA_OK;
}

int vsa_gather_tokens(const void* src, void* dst, const int64_t* slot_token, int64_t n_tokens,
                      int64_t n_slots, int64_t groups, int D, void* stream) {
  if (!src || !dst || !slot_token || n_tokens < 0 || n_slots < 0 || groups < 0)
    return VSA_ERR_INVALID_ARG;
  if (D <= 0 || D % 8) return VSA_ERR_UNSUPPORTED;
  if (!aligned16(src) || !aligned16(dst)) return VSA_ERR_INVALID_ARG;
  return launch_gather_tokens(src, dst, slot_token, n_tokens, n_slots, groups, D, false,
                              static_cast<cudaStream_t>(stream));
}

int vsa_scatter_tokens(const void* src, void* dst, const int64_t* slot_token, int64_t n_tokens,
                       int64_t n_slots, int64_t groups, int D, void* stream) {
  if (!src || !dst || !slot_token || n_tokens < 0 || n_slots < 0 || groups < 0)
    return VSA_ERR_INVALID_ARG;
  if (D <= 0 || D % 8) return VSA_ERR_UNSUPPORTED;
  if (!aligned16(src) || !aligned16(dst)) return VSA_ERR_INVALID_ARG;
  return launch_gather_tokens(src, dst, slot_token, n_tokens, n_slots, groups, D, true,
                              static_cast<cudaStream_t>(stream));
}

int vsa_set_profile_events(void* const* events) {
  if (!events) {
    g_prof_on = false;
    return VSA_OK;
  }
  for (int i = 0; i < 4; ++i) {
    if (!events[i]) return VSA_ERR_INVALID_ARG;
  }
  for (int i = 0; i < 4; ++i) g_prof_events[i] = static_cast<cudaEvent_t>(events[i]);
  g_prof_on = true;
  return VSA_OK;
}

int vsa_selftest_exp2(const float* x, float* y, int64_t n, int* mismatch, void* stream) {
  if (n < 0 || (n > 0 && (!x || !y || !mismatch))) return VSA_ERR_INVALID_ARG;
  if (n > (int64_t)1 << 40) return VSA_ERR_UNSUPPORTED;
  return launch_selftest_exp2(x, y, (long long)n, mismatch, static_cast<cudaStream_t>(stream));
}

int vsa_selftest_umma(int mode, int D, const void* a, const void* b, float* c, void* stream) {
  if (!a || !b || !c || mode < 0 || mode > 3) return VSA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return VSA_ERR_UNSUPPORTED;
  if (mode >= 2) return launch_selftest128(mode, D, a, b, c, static_cast<cudaStream_t>(stream));
  return launch_selftest_umma(mode, D, a, b, c, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
