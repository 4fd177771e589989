// vsa_forward_host: the whole VSA forward on tensors that live in host
// memory.  The inputs are staged into a caller-supplied device workspace in
// chunks of heads and the outputs copied back per chunk, so that for
// consecutive chunks the host->device copies, the kernels and the
// device->host copies run at the same time (two slots, double-buffered):
//
//   copy-in stream   : in(0)  in(1)  in(2)  ...        (waits: slot free)
//   caller's stream  :        fwd(0) fwd(1) fwd(2) ... (waits: in(i))
//   copy-out stream  :               out(0) out(1) ... (waits: fwd(i))
//
// The per-chunk forward is vsa_forward itself on a batch of one and the
// chunk's heads, so every result equals the single-call result bit for bit
// (each (batch, head) is computed independently of the others).
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <mutex>

#include "vsa.h"
#include "vsa_launch.h"

namespace vsa {
namespace {

inline size_t a256(size_t x) { return (x + 255) & ~size_t(255); }

#ifndef VSA_HOST_CHUNKS
#define VSA_HOST_CHUNKS 8
#endif
// Heads per chunk: about VSA_HOST_CHUNKS chunks in all, at least one head.
int resolve_chunk_heads(int B, int H, int heads_per_chunk) {
  if (heads_per_chunk > 0) return heads_per_chunk < H ? heads_per_chunk : H;
  if (B >= VSA_HOST_CHUNKS) return H;
  const int per_batch = (VSA_HOST_CHUNKS + B - 1) / B;  // chunks wanted per batch entry
  const int hc = (H + per_batch - 1) / per_batch;
  return hc < 1 ? 1 : hc;
}

// Byte sizes of one slot's regions for `hc` heads.
struct SlotPlan {
  size_t q, kv, gate, out, idx, num, outc, fwd, total;
  SlotPlan(int hc, int nq, int nkv, int D, int idx_stride, bool gated) {
    const size_t sq = 64u * (size_t)nq, skv = 64u * (size_t)nkv;
    q = a256((size_t)hc * sq * D * 2);
    kv = a256((size_t)hc * skv * D * 2);
    gate = gated ? a256(sq * (size_t)hc * D * 2) : 0;
    out = a256((size_t)hc * sq * D * 2);
    idx = a256((size_t)hc * nq * idx_stride * 4);
    num = a256((size_t)hc * nq * 4);
    outc = a256((size_t)hc * nq * D * 4);
    fwd = a256(vsa_forward_workspace_size(1, hc, nq, nkv, D));
    total = q + 2 * kv + gate + out + idx + num + outc + fwd;
  }
};

// The two copy streams of each device, created on first use and kept.
int copy_streams(cudaStream_t* in, cudaStream_t* out) {
  static std::mutex mu;
  static cudaStream_t s_in[64] = {nullptr}, s_out[64] = {nullptr};
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return VSA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  if (!s_in[dev] && cudaStreamCreateWithFlags(&s_in[dev], cudaStreamNonBlocking) != cudaSuccess)
    return VSA_ERR_CUDA;
  if (!s_out[dev] && cudaStreamCreateWithFlags(&s_out[dev], cudaStreamNonBlocking) != cudaSuccess)
    return VSA_ERR_CUDA;
  *in = s_in[dev];
  *out = s_out[dev];
  return VSA_OK;
}

// Events of one call: destroyed when the call has enqueued everything (the
// runtime releases an event still pending once the device reaches it).
struct CallEvents {
  cudaEvent_t start = nullptr, in_done[2] = {nullptr, nullptr}, fwd_done[2] = {nullptr, nullptr},
              out_done[2] = {nullptr, nullptr};
  bool ok = true;
  CallEvents() {
    cudaEvent_t* all[7] = {&start, &in_done[0], &in_done[1], &fwd_done[0], &fwd_done[1],
                           &out_done[0], &out_done[1]};
    for (cudaEvent_t* e : all)
      if (cudaEventCreateWithFlags(e, cudaEventDisableTiming) != cudaSuccess) ok = false;
  }
  ~CallEvents() {
    cudaEvent_t all[7] = {start, in_done[0], in_done[1], fwd_done[0], fwd_done[1], out_done[0],
                          out_done[1]};
    for (cudaEvent_t e : all)
      if (e) cudaEventDestroy(e);
  }
};

}  // namespace
}  // namespace vsa

using namespace vsa;

extern "C" size_t vsa_forward_host_workspace_size(int B, int H, int n_q_blocks, int n_kv_blocks,
                                                  int D, int idx_stride, int gated,
                                                  int heads_per_chunk) {
  if (B <= 0 || H <= 0 || n_q_blocks <= 0 || n_kv_blocks <= 0 || D <= 0 || idx_stride <= 0)
    return 0;
  const int hc = resolve_chunk_heads(B, H, heads_per_chunk);
  const SlotPlan sp(hc, n_q_blocks, n_kv_blocks, D, idx_stride, gated != 0);
  return a256(4 * ((size_t)n_q_blocks + n_kv_blocks)) + 2 * sp.total;
}

extern "C" int vsa_forward_host(const void* q, const void* k, const void* v, const void* gate,
                                const int32_t* q_block_sizes, const int32_t* kv_block_sizes,
                                int B, int H, int Sq_pad, int Skv_pad, int D, int topk,
                                float scale, void* out, int32_t* q2k_idx, int32_t* q2k_num,
                                int idx_stride, float* out_c, int heads_per_chunk,
                                void* workspace, size_t workspace_bytes, void* stream) {
  if (!q || !k || !v || !out) return VSA_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || Sq_pad <= 0 || Skv_pad <= 0 || topk < 1 || !(scale == scale) ||
      idx_stride <= 0 || heads_per_chunk < 0)
    return VSA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return VSA_ERR_UNSUPPORTED;
  if (Sq_pad % 64 || Skv_pad % 64) return VSA_ERR_SHAPE;
  const int nq = Sq_pad / 64, nkv = Skv_pad / 64;
  if (nq > VSA_MAX_BLOCKS || nkv > VSA_MAX_BLOCKS) return VSA_ERR_UNSUPPORTED;
  const int k_eff = topk < nkv ? topk : nkv;
  if (idx_stride < k_eff) return VSA_ERR_SHAPE;
  const bool gated = gate != nullptr;
  const size_t need = vsa_forward_host_workspace_size(B, H, nq, nkv, D, idx_stride, gated ? 1 : 0,
                                                      heads_per_chunk);
  if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return VSA_ERR_WORKSPACE;

  const int hc = resolve_chunk_heads(B, H, heads_per_chunk);
  const SlotPlan sp(hc, nq, nkv, D, idx_stride, gated);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaStream_t s_in = nullptr, s_out = nullptr;
  int rc = copy_streams(&s_in, &s_out);
  if (rc != VSA_OK) return rc;
  CallEvents ev;
  if (!ev.ok) return VSA_ERR_CUDA;

  // workspace: block sizes, then two slots
  char* ws = static_cast<char*>(workspace);
  int32_t* qbs_d = reinterpret_cast<int32_t*>(ws);
  int32_t* kvbs_d = qbs_d + nq;
  char* slot_base[2];
  slot_base[0] = ws + a256(4 * ((size_t)nq + nkv));
  slot_base[1] = slot_base[0] + sp.total;

#define VSA_CK(x)                                   \
  do {                                              \
    if ((x) != cudaSuccess) return VSA_ERR_CUDA;    \
  } while (0)

  // everything queued on the caller's stream so far (an earlier user of the
  // workspace, for instance) comes first
  VSA_CK(cudaEventRecord(ev.start, st));
  VSA_CK(cudaStreamWaitEvent(s_in, ev.start, 0));
  if (q_block_sizes && stage_copy_h2d(qbs_d, q_block_sizes, 4 * (size_t)nq, s_in) != VSA_OK)
    return VSA_ERR_CUDA;
  if (kv_block_sizes && stage_copy_h2d(kvbs_d, kv_block_sizes, 4 * (size_t)nkv, s_in) != VSA_OK)
    return VSA_ERR_CUDA;

  const size_t sq = (size_t)Sq_pad, skv = (size_t)Skv_pad;
  const char* qh = static_cast<const char*>(q);
  const char* kh = static_cast<const char*>(k);
  const char* vh = static_cast<const char*>(v);
  const char* gh = static_cast<const char*>(gate);
  char* oh = static_cast<char*>(out);
  const int chunks_per_b = (H + hc - 1) / hc;
  const int n_chunks = B * chunks_per_b;
  for (int c = 0; c < n_chunks; ++c) {
    const int s = c & 1;
    const int b = c / chunks_per_b;
    const int h0 = (c % chunks_per_b) * hc;
    const int nh = (H - h0) < hc ? (H - h0) : hc;
    const size_t g0 = (size_t)b * H + h0;  // first (batch, head) group of the chunk
    char* p = slot_base[s];
    char* q_d = p;
    char* k_d = q_d + sp.q;
    char* v_d = k_d + sp.kv;
    char* g_d = v_d + sp.kv;
    char* o_d = g_d + sp.gate;
    int32_t* idx_d = reinterpret_cast<int32_t*>(o_d + sp.out);
    int32_t* num_d = reinterpret_cast<int32_t*>(reinterpret_cast<char*>(idx_d) + sp.idx);
    float* oc_d = reinterpret_cast<float*>(reinterpret_cast<char*>(num_d) + sp.num);
    char* fwd_ws = reinterpret_cast<char*>(oc_d) + sp.outc;

    // copy in, once the slot's previous outputs have left
    if (c >= 2) VSA_CK(cudaStreamWaitEvent(s_in, ev.out_done[s], 0));
    VSA_CK(cudaMemcpyAsync(q_d, qh + g0 * sq * D * 2, (size_t)nh * sq * D * 2, cudaMemcpyHostToDevice, s_in));
    VSA_CK(cudaMemcpyAsync(k_d, kh + g0 * skv * D * 2, (size_t)nh * skv * D * 2, cudaMemcpyHostToDevice, s_in));
    VSA_CK(cudaMemcpyAsync(v_d, vh + g0 * skv * D * 2, (size_t)nh * skv * D * 2, cudaMemcpyHostToDevice, s_in));
    if (gated) {
      // gate [B, Sq, H, D]: the chunk's heads are nh * D contiguous values in each of Sq rows
      VSA_CK(cudaMemcpy2DAsync(g_d, (size_t)nh * D * 2, gh + ((size_t)b * sq * H + h0) * D * 2,
                               (size_t)H * D * 2, (size_t)nh * D * 2, sq, cudaMemcpyHostToDevice, s_in));
    }
    VSA_CK(cudaEventRecord(ev.in_done[s], s_in));

    // the forward of the chunk on the caller's stream
    VSA_CK(cudaStreamWaitEvent(st, ev.in_done[s], 0));
    rc = vsa_forward(q_d, k_d, v_d, gated ? g_d : nullptr, q_block_sizes ? qbs_d : nullptr,
                     kv_block_sizes ? kvbs_d : nullptr, 1, nh, Sq_pad, Skv_pad, D, topk, scale, o_d,
                     idx_d, num_d, idx_stride, out_c ? oc_d : nullptr, fwd_ws, sp.fwd, st);
    if (rc != VSA_OK) return rc;
    VSA_CK(cudaEventRecord(ev.fwd_done[s], st));

    // copy out
    VSA_CK(cudaStreamWaitEvent(s_out, ev.fwd_done[s], 0));
    VSA_CK(cudaMemcpyAsync(oh + g0 * sq * D * 2, o_d, (size_t)nh * sq * D * 2, cudaMemcpyDeviceToHost, s_out));
    if (q2k_idx)
      VSA_CK(cudaMemcpyAsync(q2k_idx + g0 * nq * idx_stride, idx_d, (size_t)nh * nq * idx_stride * 4,
                             cudaMemcpyDeviceToHost, s_out));
    if (q2k_num)
      VSA_CK(cudaMemcpyAsync(q2k_num + g0 * nq, num_d, (size_t)nh * nq * 4, cudaMemcpyDeviceToHost, s_out));
    if (out_c)
      VSA_CK(cudaMemcpyAsync(out_c + g0 * nq * D, oc_d, (size_t)nh * nq * D * 4, cudaMemcpyDeviceToHost, s_out));
    VSA_CK(cudaEventRecord(ev.out_done[s], s_out));
  }
  // the call is complete on the caller's stream once both slots' outputs are out
  for (int s = 0; s < 2 && s < n_chunks; ++s) VSA_CK(cudaStreamWaitEvent(st, ev.out_done[s], 0));
#undef VSA_CK
  return VSA_OK;
}
