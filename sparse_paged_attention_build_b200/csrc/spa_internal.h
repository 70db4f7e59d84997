// Launchers shared between the C ABI (api.cu) and the kernel files. Host
// validation happens in api.cu; these only enqueue work.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace spa {

// SM count of the current device (cached per device).
int device_sm_count();

constexpr int kSetsQueriesPerCta = 8;      // fewest queries a set-builder CTA owns
constexpr int kMaxTopkWidth = 2048;
// widest top-k row whose groups the attention's resolver sorts itself
constexpr int kInlineTopkMaxWidth = 512;

size_t build_kv_sets_workspace_bytes(int32_t n_queries);
cudaError_t launch_build_kv_sets(const int32_t* pos, int32_t n, int32_t window, int32_t ratio,
                                 const int32_t* topk, int32_t topk_width, int32_t* indptr,
                                 int32_t* indices, int64_t capacity, void* ws,
                                 uint32_t* dev_status, cudaStream_t stream);

// Fixed-scratch variant of the set builder (no caller workspace).
constexpr int32_t kNoAllocMaxQueries = 1 << 20;
size_t no_alloc_scratch_bytes();
cudaError_t launch_build_kv_sets_no_alloc(const int32_t* pos, int32_t n, int32_t window, int32_t ratio,
                                          const int32_t* topk, int32_t topk_width, int32_t* indptr,
                                          int32_t* indices, int64_t capacity, uint32_t* dev_status,
                                          cudaStream_t stream);

cudaError_t launch_paged_kv_write(const uint16_t* k_new, const uint16_t* v_new, int32_t n_tokens,
                                  int32_t head_dim, const int32_t* req, const int32_t* pos, const int32_t* pt,
                                  int32_t pt_cols, int32_t n_requests, int32_t page_size, int64_t num_pages,
                                  uint16_t* k_pool, uint16_t* v_pool, uint32_t* dev_status, cudaStream_t stream);
cudaError_t launch_unpack_d512_pages(const uint8_t* src, int64_t num_pages, int32_t page_size,
                                     const int32_t* page_ids, int32_t n_page_ids, uint16_t* dst,
                                     uint32_t* dev_status, cudaStream_t stream);
cudaError_t launch_dequant_fp8_pages(const uint8_t* src, const float* scales, int64_t num_pages,
                                     int32_t page_size, int32_t head_dim, const int32_t* page_ids,
                                     int32_t n_page_ids, bool fnuz, uint16_t* dst, uint32_t* dev_status,
                                     cudaStream_t stream);

struct AttnArgs {
  const uint16_t* q;
  int64_t q_stride_tok, q_stride_head;  // elements
  int32_t n_queries, num_heads, head_dim;
  const uint16_t *k_raw, *v_raw;
  int64_t raw_num_pages;
  int32_t raw_page_size;
  const int32_t* pt_raw;
  int32_t pt_raw_cols;
  const uint16_t *k_cmp, *v_cmp;
  // FP8 compressed pool (fused decode): codes [pages, page_size, d] and
  // FP32 scales [pages, page_size, d / 64]; when set, k_cmp/v_cmp are unused
  const uint8_t *k_cmp_fp8 = nullptr, *v_cmp_fp8 = nullptr;
  const float *k_cmp_scale = nullptr, *v_cmp_scale = nullptr;
  bool fp8_fnuz = false;   // the codes are E4M3 FNUZ rather than OCP E4M3
  int64_t cmp_num_pages;
  int32_t cmp_page_size;
  const int32_t* pt_cmp;
  int32_t pt_cmp_cols;
  const int32_t* req;
  int32_t n_requests;
  const int32_t* indptr;
  const int32_t* indices;
  // sets built inside the kernel (NULL: read indptr/indices): positions,
  // window W and ratio, and the top-k rows [n_queries, set_topk_width]
  // (NULL: every complete group); the set is the complete groups, sorted,
  // then the window
  const int32_t* set_pos = nullptr;
  int32_t set_window = 0, set_ratio = 0;
  const int32_t* set_topk = nullptr;
  int32_t set_topk_width = 0;
  const float* sink;
  float scale;
  uint16_t* out;
  float* lse;
  int32_t num_splits;  // >= 1, resolved
  void* workspace;
  uint32_t* dev_status;
  // backward only: the forward's saved O [N, H, d] BF16 and LSE [N, H], the
  // output gradient dO [N, H, d] BF16, and the FP32 gradients it adds into
  // (dq [N, H, d]; dk/dv shaped like their pools; dsink [H], may be NULL)
  const uint16_t* o_saved = nullptr;
  const float* lse_saved = nullptr;
  const uint16_t* dout = nullptr;
  float *dq = nullptr, *dk_raw = nullptr, *dv_raw = nullptr, *dk_cmp = nullptr, *dv_cmp = nullptr;
  float* dsink = nullptr;
};

constexpr int kAttnKeysPerTile = 64;
constexpr int kAttnMaxSplits = 16;
// up to this many slices merge inside one thread-block cluster (portable
// cluster size); more slices use FP32 partials in the workspace
constexpr int kAttnMaxClusterSplits = 8;
size_t attn_workspace_bytes(int32_t n_queries, int32_t num_heads, int32_t head_dim,
                            int32_t num_splits);
cudaError_t launch_sparse_sink_attn(const AttnArgs& a, cudaStream_t stream);
// Limit (ns) of the waits between the warp roles of the attention forward
// (1 s), and the testing stall: when set, every CTA of the next forward
// launches waits on a barrier nothing arrives at, with the stall's limit.
constexpr uint64_t kWaitTimeoutNsHost = 1000ull * 1000ull * 1000ull;
uint64_t attn_wait_limit_ns();
bool attn_stall();
void set_attn_stall_ns(uint64_t ns);
cudaError_t launch_sparse_sink_attn_bwd(const AttnArgs& a, cudaStream_t stream);
// head_dim 512 (32 heads per tile, transposed products); slices merge in a
// cluster only (at most kAttnMaxClusterSplits), no workspace
cudaError_t launch_sparse_sink_attn_d512(const AttnArgs& a, cudaStream_t stream);
int d512_default_splits(int32_t n_queries, int32_t num_heads);

}  // namespace spa
