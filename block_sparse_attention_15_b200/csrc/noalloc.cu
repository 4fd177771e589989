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
#include <stdint.h>

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

}  // namespace vsa

using namespace vsa;

extern "C" int vsa_forward_noalloc(const void* q, const void* k, const void* v, const void* gate,
                                   const int32_t* q_block_sizes, const int32_t* kv_block_sizes,
                                   int B, int H, int Sq_pad, int Skv_pad, int D, int topk,
                                   float scale, void* out, int32_t* q2k_idx, int32_t* q2k_num,
                                   int idx_stride, float* out_c, void* stream) {
  ForwardArgs a;
  a.block = 64;
  a.q = q; a.k = k; a.v = v; a.gate = gate;
  a.q_st = a.out_st = bhsd_strides(H, Sq_pad, D);
  a.k_st = a.v_st = bhsd_strides(H, Skv_pad, D);
  a.gate_st = gate_strides(H, Sq_pad, D);
  a.q_block_sizes = q_block_sizes; a.kv_block_sizes = kv_block_sizes;
  a.B = B; a.H = H; a.Sq_pad = Sq_pad; a.Skv_pad = Skv_pad; a.D = D; a.topk = topk;
  a.scale = scale; a.out = out; a.q2k_idx = q2k_idx; a.q2k_num = q2k_num;
  a.idx_stride = idx_stride; a.out_c = out_c;
  int rc = check_forward_args(a);
  if (rc != VSA_OK) return rc;
  // the scratch plan is vsa_forward's workspace; it must fit the array
  const size_t need = vsa_forward_workspace_size(B, H, Sq_pad / 64, Skv_pad / 64, D);
  if (need > (size_t)VSA_NOALLOC_SCRATCH_BYTES) return VSA_ERR_WORKSPACE;
  void* base = nullptr;
  rc = noalloc_scratch_address(&base);
  if (rc != VSA_OK) return rc;
  // Same launches as vsa_forward, on the fixed array.  Every region of it is
  // written in full by the kernel that produces it before any kernel reads
  // it, so nothing left over from an earlier call is used and nothing has to
  // be cleared first.
  return launch_forward(a, base, /*profile=*/false, static_cast<cudaStream_t>(stream));
}
