// The C ABI of libspa.so (declared in include/spa.h): host-side argument
// validation, workspace sizing and launch. Every failing clause returns
// before anything is enqueued and leaves a message for
// spa_last_error_detail(). No call allocates, frees or synchronises.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>

#include "spa.h"
#include "spa_internal.h"

namespace {

thread_local char g_detail[256] = "";

int fail(int status, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_detail, sizeof g_detail, fmt, ap);
  va_end(ap);
  return status;
}

int ok() {
  g_detail[0] = '\0';
  return SPA_OK;
}

int cuda_status(cudaError_t err, const char* what) {
  if (err == cudaSuccess) return ok();
  return fail(SPA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(err));
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool pow2_in(int32_t v, int32_t lo, int32_t hi) { return v >= lo && v <= hi && (v & (v - 1)) == 0; }

int32_t resolve_splits(int32_t n_queries, int32_t num_heads, int32_t requested) {
  if (requested > 0) return requested;
  return spa_sparse_sink_attn_choose_splits(n_queries, num_heads, 0);
}

}  // namespace

namespace spa {

// SM count of the current device, looked up once per device (148 if the
// query fails). Each device has its own slot, written at most once with
// the same value, so concurrent callers on different threads agree.
int device_sm_count() {
  constexpr int kSlots = 64;
  static std::atomic<int> cache[kSlots];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev >= 0 && dev < kSlots) {
    const int c = cache[dev].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  if (dev >= 0 && dev < kSlots) cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

// 0: normal launches; otherwise every CTA stalls on a barrier nothing
// arrives at, and every wait between the roles uses this limit (ns)
std::atomic<uint64_t> g_attn_stall_ns{0};
uint64_t attn_wait_limit_ns() {
  const uint64_t v = g_attn_stall_ns.load(std::memory_order_relaxed);
  return v != 0 ? v : kWaitTimeoutNsHost;
}
bool attn_stall() { return g_attn_stall_ns.load(std::memory_order_relaxed) != 0; }
void set_attn_stall_ns(uint64_t ns) { g_attn_stall_ns.store(ns, std::memory_order_relaxed); }

}  // namespace spa

extern "C" {

int spa_abi_version(void) { return SPA_ABI_VERSION; }

const char* spa_status_string(int status) {
  switch (status) {
    case SPA_OK: return "ok";
    case SPA_ERR_INVALID_ARG: return "invalid argument";
    case SPA_ERR_UNSUPPORTED: return "unsupported shape or format";
    case SPA_ERR_CAPACITY: return "output capacity too small";
    case SPA_ERR_WORKSPACE: return "workspace missing or too small";
    case SPA_ERR_ALIGNMENT: return "pointer or stride not 16-byte aligned";
    case SPA_ERR_CUDA: return "CUDA runtime error";
    default: return "unknown status";
  }
}

const char* spa_last_error_detail(void) { return g_detail; }

void spa_testing_stall_attention(uint64_t limit_ns) { spa::set_attn_stall_ns(limit_ns); }

// ---------------------------------------------------------------- sets
int64_t spa_kv_sets_capacity(int32_t n_queries, int32_t window, int32_t ratio, int32_t topk_width,
                             int32_t has_topk, int32_t max_pos) {
  if (n_queries <= 0 || window < 1 || max_pos < 0) return 0;
  const int64_t win = std::min<int64_t>(window, static_cast<int64_t>(max_pos) + 1);
  int64_t groups = 0;
  if (ratio > 0) {
    groups = (static_cast<int64_t>(max_pos) + 1) / ratio;
    if (has_topk) groups = std::min<int64_t>(groups, topk_width);
  }
  return static_cast<int64_t>(n_queries) * (win + groups);
}

size_t spa_build_kv_sets_workspace_size(int32_t n_queries) {
  return n_queries < 0 ? 0 : spa::build_kv_sets_workspace_bytes(n_queries);
}

int spa_build_kv_sets(const int32_t* pos, int32_t n_queries, int32_t window, int32_t ratio,
                      const int32_t* topk, int32_t topk_width, int32_t* indptr, int32_t* indices,
                      int64_t capacity, void* workspace, size_t workspace_bytes,
                      uint32_t* dev_status, spa_stream_t stream) {
  if (n_queries < 0) return fail(SPA_ERR_INVALID_ARG, "n_queries < 0");
  if (window < 1) return fail(SPA_ERR_INVALID_ARG, "window < 1");
  if (ratio != 0 && ratio != 4 && ratio != 128) return fail(SPA_ERR_INVALID_ARG, "ratio must be 0, 4 or 128");
  if (topk_width < 0) return fail(SPA_ERR_INVALID_ARG, "topk_width < 0");
  if (capacity < 0) return fail(SPA_ERR_INVALID_ARG, "capacity < 0");
  if (indptr == nullptr) return fail(SPA_ERR_INVALID_ARG, "indptr is NULL");
  if (n_queries > 0 && pos == nullptr) return fail(SPA_ERR_INVALID_ARG, "pos is NULL");
  if (n_queries > 0 && capacity > 0 && indices == nullptr) return fail(SPA_ERR_INVALID_ARG, "indices is NULL");
  if (ratio > 0 && topk != nullptr && topk_width > spa::kMaxTopkWidth)
    return fail(SPA_ERR_UNSUPPORTED, "topk_width > %d", spa::kMaxTopkWidth);
  if (!aligned(pos, 4) || !aligned(topk, 4) || !aligned(indptr, 4) || !aligned(indices, 4))
    return fail(SPA_ERR_ALIGNMENT, "int32 arrays must be 4-byte aligned");
  if (n_queries > 0) {
    const size_t need = spa::build_kv_sets_workspace_bytes(n_queries);
    if (workspace == nullptr || workspace_bytes < need)
      return fail(SPA_ERR_WORKSPACE, "workspace needs %zu bytes", need);
    if (!aligned(workspace, 16)) return fail(SPA_ERR_ALIGNMENT, "workspace must be 16-byte aligned");
  }
  return cuda_status(spa::launch_build_kv_sets(pos, n_queries, window, ratio, topk, topk_width, indptr,
                                               indices, capacity, workspace, dev_status,
                                               reinterpret_cast<cudaStream_t>(stream)),
                     "build_kv_sets launch");
}

// For callers that cannot allocate device memory: the same sets as
// spa_build_kv_sets, with the scan scratch taken from a fixed array inside
// the library instead of a caller workspace.
int spa_build_kv_sets_noalloc(const int32_t* pos, int32_t n_queries, int32_t window, int32_t ratio,
                              const int32_t* topk, int32_t topk_width, int32_t* indptr, int32_t* indices,
                              int64_t capacity, uint32_t* dev_status, spa_stream_t stream) {
  if (n_queries < 0) return fail(SPA_ERR_INVALID_ARG, "n_queries < 0");
  if (n_queries > spa::kNoAllocMaxQueries)
    return fail(SPA_ERR_UNSUPPORTED,
                "n_queries %d exceeds the fixed scratch of spa_build_kv_sets_noalloc (%d queries); "
                "call spa_build_kv_sets with a workspace instead",
                n_queries, spa::kNoAllocMaxQueries);
  if (window < 1) return fail(SPA_ERR_INVALID_ARG, "window < 1");
  if (ratio != 0 && ratio != 4 && ratio != 128) return fail(SPA_ERR_INVALID_ARG, "ratio must be 0, 4 or 128");
  if (topk_width < 0) return fail(SPA_ERR_INVALID_ARG, "topk_width < 0");
  if (capacity < 0) return fail(SPA_ERR_INVALID_ARG, "capacity < 0");
  if (indptr == nullptr) return fail(SPA_ERR_INVALID_ARG, "indptr is NULL");
  if (n_queries > 0 && pos == nullptr) return fail(SPA_ERR_INVALID_ARG, "pos is NULL");
  if (n_queries > 0 && capacity > 0 && indices == nullptr) return fail(SPA_ERR_INVALID_ARG, "indices is NULL");
  if (ratio > 0 && topk != nullptr && topk_width > spa::kMaxTopkWidth)
    return fail(SPA_ERR_UNSUPPORTED, "topk_width > %d", spa::kMaxTopkWidth);
  if (!aligned(pos, 4) || !aligned(topk, 4) || !aligned(indptr, 4) || !aligned(indices, 4))
    return fail(SPA_ERR_ALIGNMENT, "int32 arrays must be 4-byte aligned");
  return cuda_status(spa::launch_build_kv_sets_no_alloc(pos, n_queries, window, ratio, topk, topk_width,
                                                        indptr, indices, capacity, dev_status,
                                                        reinterpret_cast<cudaStream_t>(stream)),
                     "build_kv_sets_noalloc launch");
}

// ---------------------------------------------------------------- dequant
int spa_dequant_fp8_pages(const uint8_t* src, const float* scales, int64_t num_pages, int32_t page_size,
                          int32_t head_dim, const int32_t* page_ids, int32_t n_page_ids,
                          int32_t fp8_format, uint16_t* dst, uint32_t* dev_status, spa_stream_t stream) {
  if (num_pages < 0) return fail(SPA_ERR_INVALID_ARG, "num_pages < 0");
  if (page_size < 1) return fail(SPA_ERR_INVALID_ARG, "page_size < 1");
  if (head_dim < 1) return fail(SPA_ERR_INVALID_ARG, "head_dim < 1");
  if (n_page_ids < 0) return fail(SPA_ERR_INVALID_ARG, "n_page_ids < 0");
  if (fp8_format != 0 && fp8_format != 1)
    return fail(SPA_ERR_INVALID_ARG, "fp8_format must be 0 (OCP E4M3) or 1 (E4M3 FNUZ)");
  if (head_dim % 64 != 0) return fail(SPA_ERR_UNSUPPORTED, "head_dim must be a multiple of 64");
  if (static_cast<int64_t>(page_size) * head_dim > (1 << 24))
    return fail(SPA_ERR_UNSUPPORTED, "page_size * head_dim too large");
  if (n_page_ids > 0 && (src == nullptr || scales == nullptr || page_ids == nullptr || dst == nullptr))
    return fail(SPA_ERR_INVALID_ARG, "src, scales, page_ids and dst must be non-NULL");
  if (!aligned(src, 16) || !aligned(dst, 16)) return fail(SPA_ERR_ALIGNMENT, "src and dst must be 16-byte aligned");
  if (!aligned(scales, 4) || !aligned(page_ids, 4)) return fail(SPA_ERR_ALIGNMENT, "scales/page_ids misaligned");
  return cuda_status(spa::launch_dequant_fp8_pages(src, scales, num_pages, page_size, head_dim, page_ids,
                                                   n_page_ids, fp8_format == 1, dst, dev_status,
                                                   reinterpret_cast<cudaStream_t>(stream)),
                     "dequant_fp8_pages launch");
}

// ---------------------------------------------------------------- attention
int spa_unpack_d512_pages(const uint8_t* src, int64_t num_pages, int32_t page_size, const int32_t* page_ids,
                          int32_t n_page_ids, uint16_t* dst, uint32_t* dev_status, spa_stream_t stream) {
  if (num_pages < 0) return fail(SPA_ERR_INVALID_ARG, "num_pages < 0");
  if (page_size < 1) return fail(SPA_ERR_INVALID_ARG, "page_size < 1");
  if (n_page_ids < 0) return fail(SPA_ERR_INVALID_ARG, "n_page_ids < 0");
  if (page_size > 4096) return fail(SPA_ERR_UNSUPPORTED, "page_size above 4096");
  if (n_page_ids > 0 && (src == nullptr || page_ids == nullptr || dst == nullptr))
    return fail(SPA_ERR_INVALID_ARG, "src, page_ids and dst must be non-NULL");
  if (!aligned(src, 8)) return fail(SPA_ERR_ALIGNMENT, "src must be 8-byte aligned");
  if (!aligned(dst, 16)) return fail(SPA_ERR_ALIGNMENT, "dst must be 16-byte aligned");
  if (!aligned(page_ids, 4)) return fail(SPA_ERR_ALIGNMENT, "page_ids misaligned");
  return cuda_status(spa::launch_unpack_d512_pages(src, num_pages, page_size, page_ids, n_page_ids, dst, dev_status,
                                                   reinterpret_cast<cudaStream_t>(stream)),
                     "unpack_d512_pages launch");
}

int spa_sparse_sink_attn_choose_splits(int32_t n_queries, int32_t num_heads, int32_t max_set_size) {
  if (n_queries <= 0 || num_heads <= 0) return 1;
  const int64_t head_tiles = (num_heads + 127) / 128;
  const int64_t units = static_cast<int64_t>(n_queries) * head_tiles;
  const int64_t slots = 2 * static_cast<int64_t>(spa::device_sm_count());   // persistent CTAs, two per SM
  int64_t s = 1;
  if (units <= slots / 2) {
    // A small batch (decode) leaves CTAs idle: cut each set into slices
    // that merge inside one cluster. Measured on B200 with sets of up to
    // 640 keys: 64 queries -> 4 slices and 128 queries -> 2 slices are
    // 6 % and 15 % faster than one, while more slices than fill one wave
    // of CTAs are slower.
    s = std::min<int64_t>(slots / units, 4);
  }
  if (max_set_size > 0) {
    // long sets: slices of at least 16 tiles (1024 keys), within one wave
    const int64_t tiles = (max_set_size + spa::kAttnKeysPerTile - 1) / spa::kAttnKeysPerTile;
    s = std::max<int64_t>(s, std::min<int64_t>(slots / units, tiles / 16));
    s = std::min<int64_t>(s, std::max<int64_t>(1, tiles));   // no empty slices
  }
  s = std::max<int64_t>(1, std::min<int64_t>(s, spa::kAttnMaxSplits));
  return static_cast<int>(s);
}

int spa_sparse_sink_attn_choose_splits_d512(int32_t n_queries, int32_t num_heads) {
  if (n_queries <= 0 || num_heads <= 0) return 1;
  return spa::d512_default_splits(n_queries, num_heads);
}

int spa_paged_kv_write(const uint16_t* k_new, const uint16_t* v_new, int32_t n_tokens, int32_t head_dim,
                       const int32_t* req, const int32_t* pos, const int32_t* pt, int32_t pt_cols,
                       int32_t n_requests, int32_t page_size, int64_t num_pages, uint16_t* k_pool,
                       uint16_t* v_pool, uint32_t* dev_status, spa_stream_t stream) {
  if (n_tokens < 0) return fail(SPA_ERR_INVALID_ARG, "n_tokens < 0");
  if (head_dim < 8 || head_dim % 8 != 0) return fail(SPA_ERR_UNSUPPORTED, "head_dim must be a multiple of 8");
  if (n_requests < 1 || pt_cols < 1) return fail(SPA_ERR_INVALID_ARG, "n_requests and pt_cols must be >= 1");
  if (num_pages < 0) return fail(SPA_ERR_INVALID_ARG, "num_pages < 0");
  if (!pow2_in(page_size, 1, 1024)) return fail(SPA_ERR_UNSUPPORTED, "page_size must be a power of two <= 1024");
  if (n_tokens == 0) return ok();
  if (k_new == nullptr || v_new == nullptr || req == nullptr || pos == nullptr || pt == nullptr ||
      k_pool == nullptr || v_pool == nullptr)
    return fail(SPA_ERR_INVALID_ARG, "k_new, v_new, req, pos, pt and the pools must be non-NULL");
  if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(k_pool, 16) || !aligned(v_pool, 16))
    return fail(SPA_ERR_ALIGNMENT, "rows and pools must be 16-byte aligned");
  if (!aligned(req, 4) || !aligned(pos, 4) || !aligned(pt, 4))
    return fail(SPA_ERR_ALIGNMENT, "32-bit arrays must be 4-byte aligned");
  return cuda_status(spa::launch_paged_kv_write(k_new, v_new, n_tokens, head_dim, req, pos, pt, pt_cols, n_requests,
                                                page_size, num_pages, k_pool, v_pool, dev_status,
                                                reinterpret_cast<cudaStream_t>(stream)),
                     "paged_kv_write launch");
}

size_t spa_sparse_sink_attn_workspace_size(int32_t n_queries, int32_t num_heads, int32_t head_dim,
                                           int32_t num_splits) {
  if (n_queries <= 0 || num_heads <= 0 || head_dim <= 0 || num_splits < 0) return 0;
  if (head_dim == 512) return 0;   // slices merge inside a cluster
  return spa::attn_workspace_bytes(n_queries, num_heads, head_dim,
                                   resolve_splits(n_queries, num_heads, num_splits));
}

}  // extern "C"

namespace {

// Checks shared by every attention entry point (shapes, pools, sets; not
// the outputs nor the compressed pool's storage). SPA_OK or a failure.
int attn_check(const spa::AttnArgs& a, int32_t requested_splits) {
  if (a.n_queries < 0) return fail(SPA_ERR_INVALID_ARG, "n_queries < 0");
  if (a.num_heads < 1) return fail(SPA_ERR_INVALID_ARG, "num_heads < 1");
  if (a.n_requests < 1) return fail(SPA_ERR_INVALID_ARG, "n_requests < 1");
  if (a.head_dim != 64 && a.head_dim != 128 && a.head_dim != 512)
    return fail(SPA_ERR_UNSUPPORTED, "head_dim must be 64, 128 or 512");
  if (a.head_dim == 512) {
    if (a.num_heads > 32 && a.num_heads % 32 != 0)
      return fail(SPA_ERR_UNSUPPORTED, "head_dim 512: num_heads above 32 must be a multiple of 32");
    if (requested_splits > spa::kAttnMaxClusterSplits)
      return fail(SPA_ERR_UNSUPPORTED, "head_dim 512: num_splits at most %d", spa::kAttnMaxClusterSplits);
  } else if (a.num_heads > 128 && a.num_heads % 128 != 0) {
    return fail(SPA_ERR_UNSUPPORTED, "num_heads above 128 must be a multiple of 128");
  }
  if (a.raw_num_pages < 0 || a.pt_raw_cols < 0) return fail(SPA_ERR_INVALID_ARG, "raw pool sizes < 0");
  if (a.raw_page_size < 1) return fail(SPA_ERR_INVALID_ARG, "raw_page_size < 1");
  if (!pow2_in(a.raw_page_size, 1, 1024))
    return fail(SPA_ERR_UNSUPPORTED, "raw_page_size must be a power of two <= 1024");
  if (a.raw_num_pages * a.raw_page_size >= 0x7fffffffLL)
    return fail(SPA_ERR_UNSUPPORTED, "raw pool holds 2^31 - 1 rows or more");
  if (a.pt_cmp != nullptr) {
    if (a.cmp_num_pages < 0 || a.pt_cmp_cols < 0) return fail(SPA_ERR_INVALID_ARG, "compressed pool sizes < 0");
    if (a.cmp_page_size < 1) return fail(SPA_ERR_INVALID_ARG, "cmp_page_size < 1");
    if (!pow2_in(a.cmp_page_size, 1, 1024))
      return fail(SPA_ERR_UNSUPPORTED, "cmp_page_size must be a power of two <= 1024");
    if (a.cmp_num_pages * a.cmp_page_size >= 0x7fffffffLL)
      return fail(SPA_ERR_UNSUPPORTED, "compressed pool holds 2^31 - 1 rows or more");
  }
  if (!(a.scale > 0.f) || !std::isfinite(a.scale)) return fail(SPA_ERR_INVALID_ARG, "scale must be finite and > 0");
  if (requested_splits < 0 || requested_splits > spa::kAttnMaxSplits)
    return fail(SPA_ERR_INVALID_ARG, "num_splits must be in [0, %d]", spa::kAttnMaxSplits);
  if (a.q_stride_tok < 0 || a.q_stride_head < 0) return fail(SPA_ERR_INVALID_ARG, "negative q stride");
  if (a.n_queries == 0) return ok();
  if (a.q == nullptr) return fail(SPA_ERR_INVALID_ARG, "q must be non-NULL");
  if (a.k_raw == nullptr || a.v_raw == nullptr || a.pt_raw == nullptr)
    return fail(SPA_ERR_INVALID_ARG, "k_raw, v_raw and pt_raw must be non-NULL");
  if (a.req == nullptr) return fail(SPA_ERR_INVALID_ARG, "req must be non-NULL");
  if (a.set_pos == nullptr && (a.indptr == nullptr || a.indices == nullptr))
    return fail(SPA_ERR_INVALID_ARG, "req, indptr and indices must be non-NULL");
  if (!aligned(a.q, 16) || (a.q_stride_tok * 2) % 16 != 0 || (a.q_stride_head * 2) % 16 != 0)
    return fail(SPA_ERR_ALIGNMENT, "q base and strides must be 16-byte multiples");
  if (!aligned(a.k_raw, 16) || !aligned(a.v_raw, 16) || !aligned(a.k_cmp, 16) || !aligned(a.v_cmp, 16) ||
      !aligned(a.k_cmp_fp8, 16) || !aligned(a.v_cmp_fp8, 16))
    return fail(SPA_ERR_ALIGNMENT, "K/V pools must be 16-byte aligned");
  if (!aligned(a.sink, 4) || !aligned(a.req, 4) || !aligned(a.indptr, 4) || !aligned(a.set_pos, 4) ||
      !aligned(a.indices, 4) || !aligned(a.pt_raw, 4) || !aligned(a.pt_cmp, 4) || !aligned(a.k_cmp_scale, 4) ||
      !aligned(a.v_cmp_scale, 4))
    return fail(SPA_ERR_ALIGNMENT, "32-bit arrays must be 4-byte aligned");
  const int32_t splits = a.head_dim == 512 ? (requested_splits > 0 ? requested_splits
                                                                    : spa::d512_default_splits(a.n_queries, a.num_heads))
                                           : resolve_splits(a.n_queries, a.num_heads, requested_splits);
  if (static_cast<int64_t>(a.n_queries) * splits > 0x7fffffffLL)
    return fail(SPA_ERR_UNSUPPORTED, "n_queries * num_splits exceeds the grid");
  return ok();
}

// The forward entry points: shared checks, outputs, workspace, launch.
int attn_run(spa::AttnArgs a, int32_t requested_splits, size_t workspace_bytes, cudaStream_t stream) {
  const int st = attn_check(a, requested_splits);
  if (st != SPA_OK || a.n_queries == 0) return st;
  if (a.out == nullptr || a.lse == nullptr) return fail(SPA_ERR_INVALID_ARG, "q, out and lse must be non-NULL");
  if (!aligned(a.out, 16)) return fail(SPA_ERR_ALIGNMENT, "out must be 16-byte aligned");
  if (!aligned(a.lse, 4)) return fail(SPA_ERR_ALIGNMENT, "32-bit arrays must be 4-byte aligned");
  if (a.head_dim == 512) {
    if (a.k_cmp_fp8 != nullptr) return fail(SPA_ERR_UNSUPPORTED, "head_dim 512: the FP8 gather takes 64 or 128");
    a.num_splits = requested_splits > 0 ? requested_splits : spa::d512_default_splits(a.n_queries, a.num_heads);
    return cuda_status(spa::launch_sparse_sink_attn_d512(a, stream), "sparse_sink_attn (d 512) launch");
  }
  const int32_t splits = resolve_splits(a.n_queries, a.num_heads, requested_splits);
  const size_t need = spa::attn_workspace_bytes(a.n_queries, a.num_heads, a.head_dim, splits);
  if (need > 0) {
    if (a.workspace == nullptr || workspace_bytes < need)
      return fail(SPA_ERR_WORKSPACE, "workspace needs %zu bytes", need);
    if (!aligned(a.workspace, 256)) return fail(SPA_ERR_ALIGNMENT, "workspace must be 256-byte aligned");
  }
  a.num_splits = splits;
  return cuda_status(spa::launch_sparse_sink_attn(a, stream), "sparse_sink_attn launch");
}

spa::AttnArgs attn_args(const uint16_t* q, int64_t q_stride_tok, int64_t q_stride_head, int32_t n_queries,
                        int32_t num_heads, int32_t head_dim, const uint16_t* k_raw, const uint16_t* v_raw,
                        int64_t raw_num_pages, int32_t raw_page_size, const int32_t* pt_raw, int32_t pt_raw_cols,
                        int64_t cmp_num_pages, int32_t cmp_page_size, const int32_t* pt_cmp, int32_t pt_cmp_cols,
                        const int32_t* req, int32_t n_requests, const int32_t* indptr, const int32_t* indices,
                        const float* sink, float scale, uint16_t* out, float* lse, void* workspace,
                        uint32_t* dev_status) {
  spa::AttnArgs a;
  a.q = q;
  a.q_stride_tok = q_stride_tok;
  a.q_stride_head = q_stride_head;
  a.n_queries = n_queries;
  a.num_heads = num_heads;
  a.head_dim = head_dim;
  a.k_raw = k_raw;
  a.v_raw = v_raw;
  a.raw_num_pages = raw_num_pages;
  a.raw_page_size = raw_page_size;
  a.pt_raw = pt_raw;
  a.pt_raw_cols = pt_raw_cols;
  a.k_cmp = nullptr;
  a.v_cmp = nullptr;
  a.cmp_num_pages = cmp_num_pages;
  a.cmp_page_size = cmp_page_size;
  a.pt_cmp = pt_cmp;
  a.pt_cmp_cols = pt_cmp_cols;
  a.req = req;
  a.n_requests = n_requests;
  a.indptr = indptr;
  a.indices = indices;
  a.sink = sink;
  a.scale = scale;
  a.out = out;
  a.lse = lse;
  a.num_splits = 0;
  a.workspace = workspace;
  a.dev_status = dev_status;
  return a;
}

// The inline-set arguments of the *_inline_sets entries (checks that need
// no device data), copied into `a`.
int inline_sets_args(spa::AttnArgs& a, const int32_t* pos, const int32_t* topk, int32_t topk_width,
                     int32_t window, int32_t ratio) {
  if (window < 1) return fail(SPA_ERR_INVALID_ARG, "window must be >= 1");
  if (ratio != 0 && ratio != 4 && ratio != 128) return fail(SPA_ERR_UNSUPPORTED, "ratio must be 0, 4 or 128");
  if (topk_width < 0) return fail(SPA_ERR_INVALID_ARG, "topk_width < 0");
  if (ratio > 0 && topk != nullptr && topk_width > spa::kInlineTopkMaxWidth)
    return fail(SPA_ERR_UNSUPPORTED, "topk_width > %d (sets built in the kernel)", spa::kInlineTopkMaxWidth);
  if (pos == nullptr && a.n_queries > 0) return fail(SPA_ERR_INVALID_ARG, "pos must be non-NULL");
  if (!aligned(topk, 4)) return fail(SPA_ERR_ALIGNMENT, "32-bit arrays must be 4-byte aligned");
  a.set_pos = pos;
  a.set_window = window;
  a.set_ratio = ratio;
  // with ratio 0 the row picks nothing: the set is the window alone
  a.set_topk = ratio > 0 ? topk : nullptr;
  a.set_topk_width = ratio > 0 && topk != nullptr ? topk_width : 0;
  return SPA_OK;
}

}  // namespace

extern "C" {

int spa_sparse_sink_attn_fwd(const uint16_t* q, int64_t q_stride_tok, int64_t q_stride_head, int32_t n_queries,
                             int32_t num_heads, int32_t head_dim, const uint16_t* k_raw, const uint16_t* v_raw,
                             int64_t raw_num_pages, int32_t raw_page_size, const int32_t* pt_raw,
                             int32_t pt_raw_cols, const uint16_t* k_cmp, const uint16_t* v_cmp,
                             int64_t cmp_num_pages, int32_t cmp_page_size, const int32_t* pt_cmp,
                             int32_t pt_cmp_cols, const int32_t* req, int32_t n_requests,
                             const int32_t* indptr, const int32_t* indices, const float* sink, float scale,
                             uint16_t* out, float* lse, int32_t num_splits, void* workspace,
                             size_t workspace_bytes, uint32_t* dev_status, spa_stream_t stream) {
  if (pt_cmp != nullptr && n_queries > 0 && (k_cmp == nullptr || v_cmp == nullptr))
    return fail(SPA_ERR_INVALID_ARG, "k_cmp/v_cmp NULL with pt_cmp set");
  spa::AttnArgs a = attn_args(q, q_stride_tok, q_stride_head, n_queries, num_heads, head_dim, k_raw, v_raw,
                              raw_num_pages, raw_page_size, pt_raw, pt_raw_cols, cmp_num_pages, cmp_page_size, pt_cmp,
                              pt_cmp_cols, req, n_requests, indptr, indices, sink, scale, out, lse, workspace,
                              dev_status);
  a.k_cmp = k_cmp;
  a.v_cmp = v_cmp;
  return attn_run(a, num_splits, workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

int spa_sparse_sink_attn_fwd_inline_sets(const uint16_t* q, int64_t q_stride_tok, int64_t q_stride_head,
                                         int32_t n_queries, int32_t num_heads, int32_t head_dim,
                                         const uint16_t* k_raw, const uint16_t* v_raw, int64_t raw_num_pages,
                                         int32_t raw_page_size, const int32_t* pt_raw, int32_t pt_raw_cols,
                                         const uint16_t* k_cmp, const uint16_t* v_cmp, int64_t cmp_num_pages,
                                         int32_t cmp_page_size, const int32_t* pt_cmp, int32_t pt_cmp_cols,
                                         const int32_t* req, int32_t n_requests, const int32_t* pos,
                                         const int32_t* topk, int32_t topk_width, int32_t window, int32_t ratio,
                                         const float* sink, float scale, uint16_t* out, float* lse,
                                         int32_t num_splits, void* workspace, size_t workspace_bytes,
                                         uint32_t* dev_status, spa_stream_t stream) {
  spa::AttnArgs a = attn_args(q, q_stride_tok, q_stride_head, n_queries, num_heads, head_dim, k_raw, v_raw,
                              raw_num_pages, raw_page_size, pt_raw, pt_raw_cols, cmp_num_pages, cmp_page_size, pt_cmp,
                              pt_cmp_cols, req, n_requests, nullptr, nullptr, sink, scale, out, lse, workspace,
                              dev_status);
  const int st = inline_sets_args(a, pos, topk, topk_width, window, ratio);
  if (st != SPA_OK) return st;
  if (ratio > 0 && n_queries > 0 && (pt_cmp == nullptr || k_cmp == nullptr || v_cmp == nullptr))
    return fail(SPA_ERR_INVALID_ARG, "ratio > 0 needs the compressed pool (k_cmp, v_cmp, pt_cmp)");
  if (pt_cmp != nullptr && n_queries > 0 && (k_cmp == nullptr || v_cmp == nullptr))
    return fail(SPA_ERR_INVALID_ARG, "k_cmp/v_cmp NULL with pt_cmp set");
  a.k_cmp = k_cmp;
  a.v_cmp = v_cmp;
  return attn_run(a, num_splits, workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

int spa_sparse_sink_attn_fwd_fp8(const uint16_t* q, int64_t q_stride_tok, int64_t q_stride_head,
                                 int32_t n_queries, int32_t num_heads, int32_t head_dim, const uint16_t* k_raw,
                                 const uint16_t* v_raw, int64_t raw_num_pages, int32_t raw_page_size,
                                 const int32_t* pt_raw, int32_t pt_raw_cols, const uint8_t* k_cmp_fp8,
                                 const uint8_t* v_cmp_fp8, const float* k_cmp_scale, const float* v_cmp_scale,
                                 int64_t cmp_num_pages, int32_t cmp_page_size, const int32_t* pt_cmp,
                                 int32_t pt_cmp_cols, int32_t fp8_format, const int32_t* req, int32_t n_requests,
                                 const int32_t* indptr, const int32_t* indices, const float* sink, float scale,
                                 uint16_t* out, float* lse, int32_t num_splits, void* workspace,
                                 size_t workspace_bytes, uint32_t* dev_status, spa_stream_t stream) {
  if (fp8_format != 0 && fp8_format != 1)
    return fail(SPA_ERR_INVALID_ARG, "fp8_format must be 0 (OCP E4M3) or 1 (E4M3 FNUZ)");
  if (pt_cmp == nullptr) return fail(SPA_ERR_INVALID_ARG, "pt_cmp must be non-NULL on the FP8 path");
  if (n_queries > 0 &&
      (k_cmp_fp8 == nullptr || v_cmp_fp8 == nullptr || k_cmp_scale == nullptr || v_cmp_scale == nullptr))
    return fail(SPA_ERR_INVALID_ARG, "FP8 codes and scales must be non-NULL");
  spa::AttnArgs a = attn_args(q, q_stride_tok, q_stride_head, n_queries, num_heads, head_dim, k_raw, v_raw,
                              raw_num_pages, raw_page_size, pt_raw, pt_raw_cols, cmp_num_pages, cmp_page_size, pt_cmp,
                              pt_cmp_cols, req, n_requests, indptr, indices, sink, scale, out, lse, workspace,
                              dev_status);
  a.k_cmp_fp8 = k_cmp_fp8;
  a.v_cmp_fp8 = v_cmp_fp8;
  a.k_cmp_scale = k_cmp_scale;
  a.v_cmp_scale = v_cmp_scale;
  a.fp8_fnuz = fp8_format == 1;
  return attn_run(a, num_splits, workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

int spa_sparse_sink_attn_fwd_fp8_inline_sets(
    const uint16_t* q, int64_t q_stride_tok, int64_t q_stride_head, int32_t n_queries, int32_t num_heads,
    int32_t head_dim, const uint16_t* k_raw, const uint16_t* v_raw, int64_t raw_num_pages, int32_t raw_page_size,
    const int32_t* pt_raw, int32_t pt_raw_cols, const uint8_t* k_cmp_fp8, const uint8_t* v_cmp_fp8,
    const float* k_cmp_scale, const float* v_cmp_scale, int64_t cmp_num_pages, int32_t cmp_page_size,
    const int32_t* pt_cmp, int32_t pt_cmp_cols, int32_t fp8_format, const int32_t* req, int32_t n_requests,
    const int32_t* pos, const int32_t* topk, int32_t topk_width, int32_t window, int32_t ratio, const float* sink,
    float scale, uint16_t* out, float* lse, int32_t num_splits, void* workspace, size_t workspace_bytes,
    uint32_t* dev_status, spa_stream_t stream) {
  spa::AttnArgs a = attn_args(q, q_stride_tok, q_stride_head, n_queries, num_heads, head_dim, k_raw, v_raw,
                              raw_num_pages, raw_page_size, pt_raw, pt_raw_cols, cmp_num_pages, cmp_page_size, pt_cmp,
                              pt_cmp_cols, req, n_requests, nullptr, nullptr, sink, scale, out, lse, workspace,
                              dev_status);
  const int st = inline_sets_args(a, pos, topk, topk_width, window, ratio);
  if (st != SPA_OK) return st;
  if (fp8_format != 0 && fp8_format != 1)
    return fail(SPA_ERR_INVALID_ARG, "fp8_format must be 0 (OCP E4M3) or 1 (E4M3 FNUZ)");
  if (pt_cmp == nullptr) return fail(SPA_ERR_INVALID_ARG, "pt_cmp must be non-NULL on the FP8 path");
  if (n_queries > 0 &&
      (k_cmp_fp8 == nullptr || v_cmp_fp8 == nullptr || k_cmp_scale == nullptr || v_cmp_scale == nullptr))
    return fail(SPA_ERR_INVALID_ARG, "FP8 codes and scales must be non-NULL");
  a.k_cmp_fp8 = k_cmp_fp8;
  a.v_cmp_fp8 = v_cmp_fp8;
  a.k_cmp_scale = k_cmp_scale;
  a.v_cmp_scale = v_cmp_scale;
  a.fp8_fnuz = fp8_format == 1;
  return attn_run(a, num_splits, workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

int spa_sparse_sink_attn_bwd(const uint16_t* q, int64_t q_stride_tok, int64_t q_stride_head, int32_t n_queries,
                             int32_t num_heads, int32_t head_dim, const uint16_t* k_raw, const uint16_t* v_raw,
                             int64_t raw_num_pages, int32_t raw_page_size, const int32_t* pt_raw,
                             int32_t pt_raw_cols, const uint16_t* k_cmp, const uint16_t* v_cmp,
                             int64_t cmp_num_pages, int32_t cmp_page_size, const int32_t* pt_cmp,
                             int32_t pt_cmp_cols, const int32_t* req, int32_t n_requests,
                             const int32_t* indptr, const int32_t* indices, const float* sink, float scale,
                             const uint16_t* out, const float* lse, const uint16_t* dout, float* dq,
                             float* dk_raw, float* dv_raw, float* dk_cmp, float* dv_cmp, float* dsink,
                             int32_t num_splits, uint32_t* dev_status, spa_stream_t stream) {
  if (pt_cmp != nullptr && n_queries > 0 && (k_cmp == nullptr || v_cmp == nullptr))
    return fail(SPA_ERR_INVALID_ARG, "k_cmp/v_cmp NULL with pt_cmp set");
  spa::AttnArgs a = attn_args(q, q_stride_tok, q_stride_head, n_queries, num_heads, head_dim, k_raw, v_raw,
                              raw_num_pages, raw_page_size, pt_raw, pt_raw_cols, cmp_num_pages, cmp_page_size, pt_cmp,
                              pt_cmp_cols, req, n_requests, indptr, indices, sink, scale, nullptr, nullptr, nullptr,
                              dev_status);
  a.k_cmp = k_cmp;
  a.v_cmp = v_cmp;
  const int st = attn_check(a, num_splits);
  if (st != SPA_OK || n_queries == 0) return st;
  if (head_dim == 512) return fail(SPA_ERR_UNSUPPORTED, "the backward takes head_dim 64 or 128");
  if (out == nullptr || lse == nullptr || dout == nullptr)
    return fail(SPA_ERR_INVALID_ARG, "out, lse and dout must be non-NULL");
  if (dq == nullptr || dk_raw == nullptr || dv_raw == nullptr)
    return fail(SPA_ERR_INVALID_ARG, "dq, dk_raw and dv_raw must be non-NULL");
  if (pt_cmp != nullptr && (dk_cmp == nullptr || dv_cmp == nullptr))
    return fail(SPA_ERR_INVALID_ARG, "dk_cmp/dv_cmp NULL with pt_cmp set");
  if (!aligned(out, 16) || !aligned(dout, 16) || !aligned(dq, 16) || !aligned(dk_raw, 16) ||
      !aligned(dv_raw, 16) || !aligned(dk_cmp, 16) || !aligned(dv_cmp, 16))
    return fail(SPA_ERR_ALIGNMENT, "out, dout, dq, dk and dv must be 16-byte aligned");
  if (!aligned(lse, 4) || !aligned(dsink, 4))
    return fail(SPA_ERR_ALIGNMENT, "32-bit arrays must be 4-byte aligned");
  a.num_splits = resolve_splits(n_queries, num_heads, num_splits);
  a.o_saved = out;
  a.lse_saved = lse;
  a.dout = dout;
  a.dq = dq;
  a.dk_raw = dk_raw;
  a.dv_raw = dv_raw;
  a.dk_cmp = dk_cmp;
  a.dv_cmp = dv_cmp;
  a.dsink = sink != nullptr ? dsink : nullptr;
  return cuda_status(spa::launch_sparse_sink_attn_bwd(a, reinterpret_cast<cudaStream_t>(stream)),
                     "sparse_sink_attn_bwd launch");
}

}  // extern "C"
