// Row permutation for the head-sharded multi-GPU path: dst rows of D bf16
// elements, indexed in dst order by four coordinates (a0, a1, a2, a3) with
// extents E, are copied from src row a0*S0 + a1*S1 + a2*S2 + a3*S3.  The
// sequence-parallel wrapper uses it for the four reshards around its two
// all-to-all exchanges (README "Compiled CUDA extensions": the fused NVLink
// Ulysses all-to-all; sequence-to-head resharding): head groups packed per
// destination rank, sequence shards gathered into one sequence, and back.
//
// HBM-bound copy: one CTA per (a0, a1, a2) (grid z, y, x) copies the E3
// rows of that group with 16-byte loads and stores, 32-bit index arithmetic
// inside the group.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "vsa.h"
#include "vsa_launch.h"

namespace vsa {

struct PermuteParams {
  const uint4* src;
  uint4* dst;
  long long E1, E2;
  int E3;
  long long S0, S1, S2, S3;
  int chunks;             // 16-byte chunks per row (D / 8)
};

__global__ void __launch_bounds__(128) permute_rows_kernel(PermuteParams p) {
  const long long a2 = blockIdx.x, a1 = blockIdx.y, a0 = blockIdx.z;
  const long long dst_row0 = ((a0 * p.E1 + a1) * p.E2 + a2) * p.E3;
  const long long src_row0 = a0 * p.S0 + a1 * p.S1 + a2 * p.S2;
  const int n = p.E3 * p.chunks;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const int a3 = i / p.chunks;
    const int ch = i - a3 * p.chunks;
    const uint4 v = __ldcs(p.src + (src_row0 + a3 * p.S3) * p.chunks + ch);
    __stcs(p.dst + dst_row0 * p.chunks + i, v);
  }
}

}  // namespace vsa

using namespace vsa;

extern "C" int vsa_permute_rows(const void* src, void* dst, const int64_t* extents,
                                const int64_t* src_strides, int D, void* stream) {
  if (!src || !dst || !extents || !src_strides) return VSA_ERR_INVALID_ARG;
  if (D <= 0 || D % 8) return VSA_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) & 15u)
    return VSA_ERR_INVALID_ARG;
  for (int i = 0; i < 4; ++i)
    if (extents[i] < 0 || src_strides[i] < 0) return VSA_ERR_INVALID_ARG;
  if (extents[0] == 0 || extents[1] == 0 || extents[2] == 0 || extents[3] == 0) return VSA_OK;
  if (extents[0] > 65535 || extents[1] > 65535 || extents[2] > 0x7FFFFFFFLL ||
      extents[3] * (D / 8) > 0x7FFFFFFFLL)
    return VSA_ERR_UNSUPPORTED;
  PermuteParams p;
  p.src = static_cast<const uint4*>(src);
  p.dst = static_cast<uint4*>(dst);
  p.E1 = extents[1];
  p.E2 = extents[2];
  p.E3 = (int)extents[3];
  p.S0 = src_strides[0];
  p.S1 = src_strides[1];
  p.S2 = src_strides[2];
  p.S3 = src_strides[3];
  p.chunks = D / 8;
  const dim3 grid((unsigned)extents[2], (unsigned)extents[1], (unsigned)extents[0]);
  permute_rows_kernel<<<grid, 128, 0, static_cast<cudaStream_t>(stream)>>>(p);
  return cudaGetLastError() == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}
