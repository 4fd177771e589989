// vsa_forward_noalloc: the full VSA forward without a caller-supplied
// workspace and without any device allocation.
//
// Who needs it: callers that must not allocate device memory while they
// run -- for example a serving loop with a fixed memory budget, where a
// cudaMalloc can synchronise the device and stall every stream, or a plugin
// whose host application owns all device memory and hands it no allocator.
// Such a caller still owns q, k, v, gate and every output; only the forward's
// scratch (pooled q/k/v and the block-resolution coarse output, fp32) lives
// in the fixed-size array below, which the library defines once.
//
// The array is part of the library's device image: every GPU on which the
// library is used holds VSA_NOALLOC_SCRATCH_BYTES for it until the process
// exits.  Host code must never hand the array's name to a kernel (on the host
// it is only a stand-in for the device symbol); the device address comes
// from cudaGetSymbolAddress, looked up once per device below.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <mutex>

#include "vsa.h"
#include "vsa_launch.h"

namespace vsa {

static __device__ __align__(256) unsigned char g_noalloc_scratch[VSA_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch on the current device.  The first call
// on a device looks it up (cudaGetSymbolAddress, which may load the library's
// device image on that device); later calls reuse the cached address.
static int noalloc_scratch_address(void** out) {
  static std::mutex mu;
  static void* cached[64] = {nullptr};
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return VSA_ERR_CUDA;
  if (dev < 0 || dev >= 64) return VSA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(mu);
  if (!cached[dev]) {
    void* ptr = nullptr;
    const cudaError_t err = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (err != cudaSuccess || ptr == nullptr) return VSA_ERR_CUDA;
    cached[dev] = ptr;
  }
  *out = cached[dev];
  return VSA_OK;
}

static inline size_t noalloc_align256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace vsa

using namespace vsa;

extern "C" int vsa_forward_noalloc(const void* q, const void* k, const void* v, const void* gate,
                                   const int32_t* q_block_sizes, const int32_t* kv_block_sizes,
                                   int B, int H, int Sq_pad, int Skv_pad, int D, int topk,
                                   float scale, void* out, int32_t* q2k_idx, int32_t* q2k_num,
                                   int idx_stride, float* out_c, void* stream) {
  if (!q || !k || !v || !out || !q2k_idx || !q2k_num) return VSA_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || Sq_pad <= 0 || Skv_pad <= 0 || topk < 1 || !(scale == scale))
    return VSA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return VSA_ERR_UNSUPPORTED;
  if (Sq_pad % 64 || Skv_pad % 64) return VSA_ERR_SHAPE;
  const int nq = Sq_pad / 64, nkv = Skv_pad / 64;
  if (nq > VSA_MAX_BLOCKS || nkv > VSA_MAX_BLOCKS) return VSA_ERR_UNSUPPORTED;
  const int k_eff = topk < nkv ? topk : nkv;
  if (idx_stride < k_eff) return VSA_ERR_SHAPE;
  const uintptr_t mis = reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
                        reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(out) |
                        reinterpret_cast<uintptr_t>(gate) | reinterpret_cast<uintptr_t>(out_c);
  if (mis & 15u) return VSA_ERR_INVALID_ARG;

  // Scratch plan, same order as vsa_forward's workspace: pooled q, pooled k,
  // pooled v, the coarse output unless the caller receives it in out_c, then
  // the block row norms and the per-query-block logit bound.
  const size_t g = (size_t)B * H * D * sizeof(float);
  const size_t G = (size_t)B * H;
  const size_t need = noalloc_align256(g * nq) * 2 + noalloc_align256(g * nkv) * 2 +
                      noalloc_align256(G * (2 * (size_t)nq + nkv) * sizeof(float));
  if (need > (size_t)VSA_NOALLOC_SCRATCH_BYTES) return VSA_ERR_WORKSPACE;  // too big for the array

  void* base = nullptr;
  int rc = noalloc_scratch_address(&base);
  if (rc != VSA_OK) return rc;
  int* status = device_status_ptr();
  if (!status) return VSA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  // Every region is written in full by the kernel that produces it before any
  // kernel reads it, so nothing left over from an earlier call is ever used
  // and nothing has to be cleared first.
  char* ws = static_cast<char*>(base);
  float* qc = reinterpret_cast<float*>(ws);
  ws += noalloc_align256(g * nq);
  float* kc = reinterpret_cast<float*>(ws);
  ws += noalloc_align256(g * nkv);
  float* vc = reinterpret_cast<float*>(ws);
  ws += noalloc_align256(g * nkv);
  float* oc = out_c ? out_c : reinterpret_cast<float*>(ws);
  ws += noalloc_align256(g * nq);
  float* qn = reinterpret_cast<float*>(ws);
  float* kn = qn + G * nq;
  float* qk_bound = kn + G * nkv;

  PoolParams pp;
  pp.q = static_cast<const __nv_bfloat16*>(q);
  pp.k = static_cast<const __nv_bfloat16*>(k);
  pp.v = static_cast<const __nv_bfloat16*>(v);
  pp.q_bs = q_block_sizes;
  pp.kv_bs = kv_block_sizes;
  pp.groups = B * H;
  pp.nq = nq;
  pp.nkv = nkv;
  pp.qc = qc;
  pp.kc = kc;
  pp.vc = vc;
  pp.qn = qn;
  pp.kn = kn;
  pp.status = status;
  rc = launch_pool(pp, D, st);
  if (rc != VSA_OK) return rc;

  const float sc = scale > 0.f ? scale : 1.0f / sqrtf((float)D);
  CoarseParams cp;
  cp.qc = qc;
  cp.kc = kc;
  cp.vc = vc;
  cp.groups = B * H;
  cp.nq = nq;
  cp.nkv = nkv;
  cp.scale = sc;
  cp.topk = k_eff;
  cp.idx_stride = idx_stride;
  cp.q2k_idx = q2k_idx;
  cp.q2k_num = q2k_num;
  cp.out_c = oc;
  cp.qn = qn;
  cp.kn = kn;
  cp.qk_bound = qk_bound;
  cp.bound_scale = sc * 1.4426950408889634f * (1.f + 0x1p-8f);
  cp.status = status;
  rc = launch_coarse_topk(cp, D, st);
  if (rc != VSA_OK) return rc;

  SparseParams sp;
  memset(&sp, 0, sizeof(sp));
  sp.out = static_cast<__nv_bfloat16*>(out);
  sp.gate = static_cast<const __nv_bfloat16*>(gate);
  sp.out_c = oc;
  sp.q2k_idx = q2k_idx;
  sp.q2k_num = q2k_num;
  sp.idx_stride = idx_stride;
  sp.q_bs = q_block_sizes;
  sp.kv_bs = kv_block_sizes;
  sp.B = B;
  sp.H = H;
  sp.nq = nq;
  sp.nkv = nkv;
  sp.q_rows_per_group = Sq_pad;
  sp.kv_rows_per_group = Skv_pad;
  sp.gate_seq = Sq_pad;
  sp.scale_log2 = sc * 1.4426950408889634f;
  sp.qk_bound = qk_bound;
  sp.varlen = 0;
  sp.status = status;
  return launch_sparse(sp, q, k, v, (long long)B * H * Sq_pad, (long long)B * H * Skv_pad, D,
                       /*combine=*/true, /*gated=*/gate != nullptr, st);
}
