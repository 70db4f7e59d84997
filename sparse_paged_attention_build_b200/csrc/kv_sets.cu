// Per-token KV sets as CSR in canonical (ascending key) order.
//
// Page "Roadmap item 24 - joint compressed/window attention with sink",
// section "Contracts and lifetime": logical request/position/kind keys,
// complete windows, C4/C128 group boundaries, canonical KV ordering. Page
// "test: add block-level DeepSeek-V4 attention test", opening section and
// "Validation": ratio 0 / 4 / 128 layers; top-k truncates only once the
// complete groups outnumber it.
//
// A CTA owns a block of consecutive queries, one warp per query at a time.
// A warp filters its top-k row (keeps 0 <= g < floor((p+1)/ratio)) into a
// shared-memory bitmap over the complete groups -- setting a bit drops
// repeats and reading the words in order yields the ascending list -- and
// counts the set bits; when the complete groups outnumber the bitmap it
// sorts the row with a bitonic network instead. The window adds min(p+1, W)
// keys. The CTA scans its counts, publishes its total and obtains its offset
// by a decoupled look-back over the CTAs before it (CTA order taken from an
// atomic ticket, so every predecessor is already running; one warp reads 32
// predecessors per step), then recomputes every set and writes its indptr
// entry and its keys: the distinct groups ascending (listed in shared
// memory, then copied out coalesced), then the window tokens ascending with
// the window tag. A warp writes its queries in the reverse of the counting
// order, so the bitmap of its first one is still in place. Integer only; no
// floating point anywhere.
#include <climits>
#include <mutex>

#include <cuda.h>

#include "spa_device.cuh"
#include "spa_internal.h"

namespace spa {
namespace {

constexpr uint64_t kFlagAggregate = 1ull << 62;
constexpr uint64_t kFlagInclusive = 2ull << 62;
constexpr uint64_t kValueMask = (1ull << 62) - 1;

__device__ __forceinline__ uint64_t ld_relaxed_u64(const uint64_t* p) {
  uint64_t v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_relaxed_u64(uint64_t* p, uint64_t v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// Ascending bitonic sort of buf[0, n) (n a power of two) by one warp.
__device__ void warp_bitonic_sort(int32_t* buf, int n, int lane) {
  for (int k = 2; k <= n; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int t = lane; t < (n >> 1); t += 32) {
        const int lo = ((t & ~(j - 1)) << 1) | (t & (j - 1));
        const int hi = lo | j;
        const bool up = (lo & k) == 0;
        const int32_t a = buf[lo], b = buf[hi];
        if ((a > b) == up) {
          buf[lo] = b;
          buf[hi] = a;
        }
      }
      __syncwarp();
    }
  }
}

struct SetsParams {
  const int32_t* pos;
  int32_t n;
  int32_t window;
  int32_t ratio;
  const int32_t* topk;
  int32_t topk_width;
  int32_t sort_width;  // topk_width rounded up to a power of two (>= 32)
  int32_t buf_words;   // per-warp shared buffer (>= sort_width), also the bitmap size
  int32_t per_cta;     // consecutive queries owned by one CTA
  int32_t* indptr;
  int32_t* indices;
  int64_t capacity;
  uint64_t* tile_status;
  uint32_t* tile_ticket;
  uint32_t* dev_status;
};

constexpr int kSetsWarps = 16;   // warps per CTA, one query each at a time
constexpr int kRowStep = 512;    // top-k entries a warp loads at once
constexpr int kRegWords = 16;    // bitmap words per lane held in registers while writing a list
constexpr int kMaxPerCta = 2048;

__device__ __forceinline__ int64_t warp_sum64(int64_t v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// The key set of query i, by one warp (all lanes call together). Returns
// the number of keys; when `write` is set, stores them at
// indices[start ..) ascending (entries at or past `limit` are dropped).
// `bitmap_ready`: buf still holds this query's bitmap from the counting
// pass (the warp's last query there is its first here).
__device__ int64_t one_query(const SetsParams& P, int64_t i, int32_t* buf, int lane, bool write,
                             int64_t start, int64_t limit, bool bitmap_ready = false) {
  const int32_t p = P.pos[i];
  if (p < 0 || p >= SPA_WINDOW_TAG) {
    if (lane == 0 && !write) report(P.dev_status, SPA_DEV_BAD_INDEX);
    return 0;
  }
  const int32_t n_window = min(p + 1, P.window);
  const int32_t n_complete = P.ratio > 0 ? (p + 1) / P.ratio : 0;
  const bool listed = P.ratio > 0 && P.topk != nullptr;
  const int words = (n_complete + 31) >> 5;
  const bool use_bitmap = listed && words <= P.buf_words;
  int64_t n_groups = 0;
  if (P.ratio > 0 && !listed) {
    n_groups = n_complete;
    if (write)
      for (int64_t g = lane; g < n_groups; g += 32)
        if (start + g < limit) P.indices[start + g] = static_cast<int32_t>(g);
  } else if (use_bitmap) {
    // bitmap over the complete groups: marking a bit removes repeats,
    // reading the words in order gives the ascending list
    uint32_t* bm = reinterpret_cast<uint32_t*>(buf);
    if (!bitmap_ready) {
      for (int w = lane; w < words; w += 32) bm[w] = 0u;
      __syncwarp();
      const int32_t* row = P.topk + i * P.topk_width;
      // 512 entries per step with all 16 loads of a lane in flight together
      // (one round trip per step rather than one per entry)
      for (int j0 = 0; j0 < P.topk_width; j0 += kRowStep) {
        int32_t g[kRowStep / 32];
#pragma unroll
        for (int r = 0; r < kRowStep / 32; ++r) {
          const int j = j0 + 32 * r + lane;
          g[r] = j < P.topk_width ? __ldg(row + j) : -1;
        }
#pragma unroll
        for (int r = 0; r < kRowStep / 32; ++r)
          if (g[r] >= 0 && g[r] < n_complete) atomicOr(bm + (g[r] >> 5), 1u << (g[r] & 31));
      }
      __syncwarp();
    }
    if (!write) {
      // counting needs only the number of set bits; the bitmap stays
      int32_t cnt = 0;
      for (int w = lane; w < words; w += 32) cnt += __popc(bm[w]);
      n_groups = warp_sum64(cnt);
    } else if (words <= 32 * kRegWords) {
      // every word into registers (word 32 r + lane in register r), then
      // the ascending list over the bitmap in shared memory and one
      // coalesced copy of it
      uint32_t m[kRegWords];
#pragma unroll
      for (int r = 0; r < kRegWords; ++r) m[r] = 32 * r + lane < words ? bm[32 * r + lane] : 0u;
      __syncwarp();
      int32_t total = 0;
#pragma unroll
      for (int r = 0; r < kRegWords; ++r) {
        if (32 * r >= words) continue;   // uniform across the warp
        const int cnt = __popc(m[r]);
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int v = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += v;
        }
        int32_t at = total + incl - cnt;
        const int32_t base = (32 * r + lane) * 32;
        for (uint32_t bits = m[r]; bits != 0u; bits &= bits - 1u) buf[at++] = base + (__ffs(bits) - 1);
        total += __shfl_sync(0xffffffffu, incl, 31);
      }
      __syncwarp();
      for (int k = lane; k < total; k += 32)
        if (start + k < limit) P.indices[start + k] = buf[k];
      n_groups = total;
    } else {
      int64_t written = 0;
      for (int w0 = 0; w0 < words; w0 += 32) {
        const int w = w0 + lane;
        uint32_t bits = w < words ? bm[w] : 0u;
        const int cnt = __popc(bits);
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int v = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += v;
        }
        int64_t dst = start + written + (incl - cnt);
        while (bits) {
          const int bit = __ffs(bits) - 1;
          if (dst < limit) P.indices[dst] = w * 32 + bit;
          ++dst;
          bits &= bits - 1u;
        }
        written += __shfl_sync(0xffffffffu, incl, 31);
      }
      n_groups = written;
    }
    __syncwarp();   // the bitmap is rebuilt by the next query
  } else if (listed) {
    const int32_t* row = P.topk + i * P.topk_width;
    for (int j0 = 0; j0 < P.sort_width; j0 += kRowStep) {
      int32_t g[kRowStep / 32];
#pragma unroll
      for (int r = 0; r < kRowStep / 32; ++r) {
        const int j = j0 + 32 * r + lane;
        g[r] = j < P.topk_width ? __ldg(row + j) : -1;
      }
#pragma unroll
      for (int r = 0; r < kRowStep / 32; ++r) {
        const int j = j0 + 32 * r + lane;
        if (j < P.sort_width) buf[j] = (g[r] >= 0 && g[r] < n_complete) ? g[r] : INT_MAX;
      }
    }
    __syncwarp();
    warp_bitonic_sort(buf, P.sort_width, lane);
    int64_t written = 0;
    for (int j0 = 0; j0 < P.sort_width; j0 += 32) {
      if (buf[j0] == INT_MAX) break;   // sentinels sort last
      const int j = j0 + lane;
      const int32_t v = buf[j];
      const bool first = v != INT_MAX && (j == 0 || buf[j - 1] != v);
      const uint32_t m = __ballot_sync(0xffffffffu, first);
      if (write) {
        const int64_t dst = start + written + __popc(m & ((1u << lane) - 1u));
        if (first && dst < limit) P.indices[dst] = v;
      }
      written += __popc(m);
    }
    n_groups = written;
    __syncwarp();
  }
  if (write) {
    const int32_t t0 = p - n_window + 1;
    for (int t = lane; t < n_window; t += 32) {
      const int64_t dst = start + n_groups + t;
      if (dst < limit) P.indices[dst] = SPA_WINDOW_TAG | (t0 + t);
    }
  }
  return n_groups + n_window;
}

// Persistent layout: CTA k (in the order of an atomic ticket, so that every
// CTA before it is already running) owns queries [k * per_cta, ...). It
// counts every owned set, scans the counts, publishes its total and finds
// its offset by a decoupled look-back whose warp reads 32 predecessors per
// step, then recomputes each set and writes it with its indptr entry.
__global__ void __launch_bounds__(kSetsWarps * 32) build_kv_sets_kernel(const SetsParams P) {
  extern __shared__ int32_t sets_smem[];   // [kSetsWarps][buf_words] | int64 prefix[per_cta]
  __shared__ int64_t s_base;
  __shared__ uint32_t s_tile;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  int32_t* buf = sets_smem + warp * P.buf_words;
  int64_t* prefix = reinterpret_cast<int64_t*>(sets_smem + kSetsWarps * P.buf_words);
  if (threadIdx.x == 0) s_tile = atomicAdd(P.tile_ticket, 1u);
  // the attention launched next may start its setup now (it waits for this
  // grid to finish before it reads the sets)
  grid_dep_launch();
  __syncthreads();
  const uint32_t tile = s_tile;
  // A ticket past this launch's grid only comes from another launch using
  // the same scratch at the same time (a shared workspace, or overlapping
  // calls of the no-allocation entry point). The status words of such a
  // tile lie outside what this launch cleared: touch none of them.
  if (tile >= gridDim.x) {
    if (threadIdx.x == 0) report(P.dev_status, SPA_DEV_SCRATCH_RACE);
    return;
  }
  const int64_t q0 = static_cast<int64_t>(tile) * P.per_cta;
  const int nq = static_cast<int>(min(static_cast<int64_t>(P.per_cta), static_cast<int64_t>(P.n) - q0));

  int last_q = -1;
  for (int q = warp; q < nq; q += kSetsWarps) {
    const int64_t c = one_query(P, q0 + q, buf, lane, false, 0, 0);
    if (lane == 0) prefix[q] = c;
    last_q = q;
  }
  __syncthreads();

  if (warp == 0) {
    // exclusive scan of the counts: a block of them per lane, then the lanes
    const int per = (nq + 31) / 32;
    const int lo = min(lane * per, nq), hi = min(lo + per, nq);
    int64_t own = 0;
    for (int q = lo; q < hi; ++q) own += prefix[q];
    int64_t incl = own;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int64_t run = incl - own;
    for (int q = lo; q < hi; ++q) {
      const int64_t v = prefix[q];
      prefix[q] = run;
      run += v;
    }
    const int64_t total = __shfl_sync(0xffffffffu, incl, 31);

    // offset of this CTA: decoupled look-back, 32 predecessors per step
    int64_t excl = 0;
    if (tile == 0) {
      if (lane == 0) st_relaxed_u64(P.tile_status, kFlagInclusive | static_cast<uint64_t>(total));
    } else {
      if (lane == 0) st_relaxed_u64(P.tile_status + tile, kFlagAggregate | static_cast<uint64_t>(total));
      int64_t top = static_cast<int64_t>(tile) - 1;
      const uint64_t t0 = global_timer_ns();
      uint32_t spins = 0;
      while (true) {
        const int64_t idx = top - lane;
        const uint64_t s = idx >= 0 ? ld_relaxed_u64(P.tile_status + idx) : kFlagInclusive;
        if (__any_sync(0xffffffffu, (s & ~kValueMask) == 0)) {   // a predecessor has not published yet
          if ((++spins & 63u) == 0 && global_timer_ns() - t0 > kWaitTimeoutNs) {
            if (lane == 0) report(P.dev_status, SPA_DEV_TIMEOUT);
            break;
          }
          continue;
        }
        const uint32_t inc = __ballot_sync(0xffffffffu, (s & ~kValueMask) == kFlagInclusive);
        const int last = inc ? __ffs(inc) - 1 : 31;   // nearest inclusive predecessor
        excl += warp_sum64(lane <= last ? static_cast<int64_t>(s & kValueMask) : 0);
        if (inc) break;
        top -= 32;
      }
      if (lane == 0)
        st_relaxed_u64(P.tile_status + tile, kFlagInclusive | static_cast<uint64_t>(excl + total));
    }
    if (lane == 0) s_base = excl;
  }
  __syncthreads();

  const int64_t base = s_base;
  const int64_t limit = P.capacity < INT_MAX ? P.capacity : INT_MAX;
  // the warp's queries in reverse order: the first one's bitmap is still
  // in its buffer from the counting pass
  for (int q = last_q; q >= 0; q -= kSetsWarps) {
    const int64_t i = q0 + q;
    const int64_t start = base + prefix[q];
    const int64_t c = one_query(P, i, buf, lane, true, start, limit, q == last_q);
    if (lane == 0) {
      const int64_t end = start + c;
      if (end > P.capacity || end > INT_MAX) report(P.dev_status, SPA_DEV_CAPACITY);
      P.indptr[i] = static_cast<int32_t>(start < INT_MAX ? start : INT_MAX);
      if (i == P.n - 1) P.indptr[P.n] = static_cast<int32_t>(end < INT_MAX ? end : INT_MAX);
    }
  }
}

int sort_width_for(int32_t topk_width) {
  int w = 32;
  while (w < topk_width) w <<= 1;
  return w;
}

}  // namespace

// An upper bound of the scratch the launcher uses (it uses fewer status
// words when a CTA owns more than kSetsQueriesPerCta queries).
size_t build_kv_sets_workspace_bytes(int32_t n_queries) {
  const int64_t tiles = (static_cast<int64_t>(n_queries) + kSetsQueriesPerCta - 1) / kSetsQueriesPerCta;
  return static_cast<size_t>(tiles) * sizeof(uint64_t) + 16;
}

namespace {

// Enqueue the set builder with its look-back status words at `tile_status`
// (one per CTA) and its CTA ticket at `ticket`; both are cleared first.
cudaError_t launch_sets(const int32_t* pos, int32_t n, int32_t window, int32_t ratio, const int32_t* topk,
                        int32_t topk_width, int32_t* indptr, int32_t* indices, int64_t capacity,
                        uint64_t* tile_status, uint32_t* ticket, bool ticket_follows_status,
                        uint32_t* dev_status, cudaStream_t stream) {
  if (n == 0) return cudaMemsetAsync(indptr, 0, sizeof(int32_t), stream);
  // about two CTAs per SM, each with a contiguous block of queries
  const int64_t slots = 2 * static_cast<int64_t>(device_sm_count());
  int64_t per_cta = (static_cast<int64_t>(n) + slots - 1) / slots;
  per_cta = per_cta < kSetsQueriesPerCta ? kSetsQueriesPerCta : (per_cta > kMaxPerCta ? kMaxPerCta : per_cta);
  const int64_t tiles = (static_cast<int64_t>(n) + per_cta - 1) / per_cta;
  const size_t status_bytes = static_cast<size_t>(tiles) * sizeof(uint64_t);
  cudaError_t err;
  if (ticket_follows_status) {   // one clear covers both
    err = cudaMemsetAsync(tile_status, 0, status_bytes + 16, stream);
  } else {
    err = cudaMemsetAsync(tile_status, 0, status_bytes, stream);
    if (err == cudaSuccess) err = cudaMemsetAsync(ticket, 0, 16, stream);
  }
  if (err != cudaSuccess) return err;
  SetsParams P;
  P.pos = pos;
  P.n = n;
  P.window = window;
  P.ratio = ratio;
  P.topk = (ratio > 0) ? topk : nullptr;
  P.topk_width = topk_width;
  P.sort_width = (P.topk != nullptr) ? sort_width_for(topk_width) : 32;
  // bitmap of at least 512 words (16384 groups) per warp; the sort handles
  // queries with more complete groups than that
  P.buf_words = (P.topk != nullptr) ? (P.sort_width > 512 ? P.sort_width : 512) : 0;
  P.per_cta = static_cast<int32_t>(per_cta);
  P.indptr = indptr;
  P.indices = indices;
  P.capacity = capacity;
  P.tile_status = tile_status;
  P.tile_ticket = ticket;
  P.dev_status = dev_status;
  const size_t smem = static_cast<size_t>(kSetsWarps) * P.buf_words * sizeof(int32_t) +
                      static_cast<size_t>(per_cta) * sizeof(int64_t);
  if (smem > 48 * 1024) {
    err = cudaFuncSetAttribute(build_kv_sets_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem));
    if (err != cudaSuccess) return err;
  }
  build_kv_sets_kernel<<<static_cast<unsigned>(tiles), kSetsWarps * 32, smem, stream>>>(P);
  return cudaGetLastError();
}

size_t sets_tiles(int32_t n) {
  const int64_t slots = 2 * static_cast<int64_t>(device_sm_count());
  int64_t per_cta = (static_cast<int64_t>(n) + slots - 1) / slots;
  per_cta = per_cta < kSetsQueriesPerCta ? kSetsQueriesPerCta : (per_cta > kMaxPerCta ? kMaxPerCta : per_cta);
  return static_cast<size_t>((static_cast<int64_t>(n) + per_cta - 1) / per_cta);
}

}  // namespace

cudaError_t launch_build_kv_sets(const int32_t* pos, int32_t n, int32_t window, int32_t ratio,
                                 const int32_t* topk, int32_t topk_width, int32_t* indptr,
                                 int32_t* indices, int64_t capacity, void* ws,
                                 uint32_t* dev_status, cudaStream_t stream) {
  uint64_t* status = static_cast<uint64_t*>(ws);
  uint32_t* ticket = reinterpret_cast<uint32_t*>(status + (n > 0 ? sets_tiles(n) : 0));
  return launch_sets(pos, n, window, ratio, topk, topk_width, indptr, indices, capacity, status, ticket, true,
                     dev_status, stream);
}

// ---------------------------------------------------------------------------
// Variant without caller workspace, for callers that cannot allocate device
// memory. The look-back status words and the CTA ticket live in a fixed
// array that every GPU loading this library keeps for the life of the
// process (kNoAllocScratchBytes, about 1 MiB).
// ---------------------------------------------------------------------------
namespace {

constexpr int64_t kNoAllocMaxTiles = (kNoAllocMaxQueries + kSetsQueriesPerCta - 1) / kSetsQueriesPerCta;
constexpr size_t kNoAllocScratchBytes = static_cast<size_t>(kNoAllocMaxTiles) * sizeof(uint64_t) + 16;
static_assert(kNoAllocScratchBytes == 1048576 + 16, "the documented limit");

static __device__ __align__(256) uint64_t g_sets_scratch[kNoAllocScratchBytes / sizeof(uint64_t)];

// Host code cannot pass &g_sets_scratch to a kernel: on the host that name
// is only a stand-in. Its device address is looked up once per device (and
// context: a device reset makes a new context and a new address), with that
// device current, and cached.
constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_ptr[kMaxDevices] = {};
unsigned long long g_scratch_ctx[kMaxDevices] = {};

// Unique id of the current context (0 if the driver cannot say).
unsigned long long current_context_id() {
  using GetCurrent = CUresult (*)(CUcontext*);
  using GetId = CUresult (*)(CUcontext, unsigned long long*);
  static GetCurrent get_current = nullptr;
  static GetId get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrent>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetId>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current == nullptr || get_id == nullptr || get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr ||
      get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

cudaError_t scratch_for_current_device(void** out) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_ptr[dev] == nullptr || g_scratch_ctx[dev] != ctx) {
    void* p = nullptr;
    err = cudaGetSymbolAddress(&p, g_sets_scratch);
    if (err != cudaSuccess) return err;
    g_scratch_ptr[dev] = p;
    g_scratch_ctx[dev] = ctx;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace

size_t no_alloc_scratch_bytes() { return kNoAllocScratchBytes; }

cudaError_t launch_build_kv_sets_no_alloc(const int32_t* pos, int32_t n, int32_t window, int32_t ratio,
                                          const int32_t* topk, int32_t topk_width, int32_t* indptr,
                                          int32_t* indices, int64_t capacity, uint32_t* dev_status,
                                          cudaStream_t stream) {
  void* scratch = nullptr;
  cudaError_t err = scratch_for_current_device(&scratch);
  if (err != cudaSuccess) return err;
  // The same kernel as the workspace entry point. The status words start
  // at the array's base; the CTA ticket sits in the array's last 16 bytes,
  // past the status words of the largest call, so that no call's ticket
  // ever lands on another call's status words. The launcher clears both
  // before the kernel runs.
  uint64_t* status = static_cast<uint64_t*>(scratch);
  uint32_t* ticket = reinterpret_cast<uint32_t*>(static_cast<char*>(scratch) + kNoAllocScratchBytes - 16);
  return launch_sets(pos, n, window, ratio, topk, topk_width, indptr, indices, capacity, status, ticket, false,
                     dev_status, stream);
}

}  // namespace spa
