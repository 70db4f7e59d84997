// New raw tokens into the paged window cache.
//
// Page "test: add block-level DeepSeek-V4 attention test", decode kernel
// timeline and its notes: the paged KV write ("swa_write", fused into the
// qk-norm + RoPE kernel in decode as "kvw_paged") puts each new token's K
// and V row into the sliding-window cache through the page table, ahead of
// the sparse attention core. Here it is the plain write, without the norm
// or RoPE that precede it in the model: token j (request b = req[j],
// position t = pos[j]) goes to row pt[b][t / page_size] * page_size +
// t % page_size of both pools.
//
// One warp per token: the K and V rows (2 * d bytes each) move in 16-byte
// pieces, coalesced on both sides. HBM-bound: 8 * d bytes per token.
#include "spa_device.cuh"
#include "spa_internal.h"

namespace spa {
namespace {

constexpr int kWriteWarps = 8;

__global__ void __launch_bounds__(kWriteWarps * 32)
paged_kv_write_kernel(const uint4* __restrict__ k_new, const uint4* __restrict__ v_new, int32_t n_tokens,
                      int32_t pieces, const int32_t* __restrict__ req, const int32_t* __restrict__ pos,
                      const int32_t* __restrict__ pt, int32_t pt_cols, int32_t n_requests, int32_t ps_log2,
                      int64_t num_pages, uint4* k_pool, uint4* v_pool, uint32_t* dev_status) {
  const int lane = threadIdx.x & 31;
  const int64_t j = static_cast<int64_t>(blockIdx.x) * kWriteWarps + (threadIdx.x >> 5);
  if (j >= n_tokens) return;
  const int32_t b = __ldg(req + j);
  const int32_t t = __ldg(pos + j);
  if (b < 0 || b >= n_requests || t < 0 || (t >> ps_log2) >= pt_cols) {
    if (lane == 0) report(dev_status, SPA_DEV_BAD_INDEX);
    return;
  }
  const int64_t page = __ldg(pt + static_cast<int64_t>(b) * pt_cols + (t >> ps_log2));
  if (page < 0 || page >= num_pages) {
    if (lane == 0) report(dev_status, SPA_DEV_BAD_PAGE);
    return;
  }
  const int64_t row = (page << ps_log2) + (t & ((1 << ps_log2) - 1));
  // the K row's pieces, then the V row's, spread over all 32 lanes
  for (int p = lane; p < 2 * pieces; p += 32) {
    const bool is_k = p < pieces;
    const int q = is_k ? p : p - pieces;
    (is_k ? k_pool : v_pool)[row * pieces + q] = __ldg((is_k ? k_new : v_new) + j * pieces + q);
  }
}

}  // namespace

cudaError_t launch_paged_kv_write(const uint16_t* k_new, const uint16_t* v_new, int32_t n_tokens,
                                  int32_t head_dim, const int32_t* req, const int32_t* pos, const int32_t* pt,
                                  int32_t pt_cols, int32_t n_requests, int32_t page_size, int64_t num_pages,
                                  uint16_t* k_pool, uint16_t* v_pool, uint32_t* dev_status, cudaStream_t stream) {
  if (n_tokens == 0) return cudaSuccess;
  int ps_log2 = 0;
  while ((1 << ps_log2) < page_size) ++ps_log2;
  const int32_t pieces = head_dim * 2 / 16;
  const unsigned blocks = static_cast<unsigned>((static_cast<int64_t>(n_tokens) + kWriteWarps - 1) / kWriteWarps);
  paged_kv_write_kernel<<<blocks, kWriteWarps * 32, 0, stream>>>(
      reinterpret_cast<const uint4*>(k_new), reinterpret_cast<const uint4*>(v_new), n_tokens, pieces, req, pos, pt,
      pt_cols, n_requests, ps_log2, num_pages, reinterpret_cast<uint4*>(k_pool), reinterpret_cast<uint4*>(v_pool),
      dev_status);
  return cudaGetLastError();
}

}  // namespace spa
