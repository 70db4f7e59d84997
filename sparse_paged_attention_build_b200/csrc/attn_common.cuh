// Pieces shared by the attention kernels (forward and backward): the chunk
// descriptors the resolver hands to the other warp roles, the resolver
// itself (keys -> physical pool rows through the page tables), and the
// host-side tensor-map encoders.
#pragma once

#include <algorithm>
#include <climits>
#include <cstdint>

#include <cuda.h>
#include <cudaTypedefs.h>

#include "spa_device.cuh"
#include "spa_internal.h"

namespace spa {
namespace attn {

constexpr int kT = kAttnKeysPerTile;             // keys per tile
constexpr int kChunkKeys = 640;                  // keys resolved per chunk (10 tiles; 768 measured slower)
constexpr uint32_t kRawBit = 0x80000000u;        // row of the raw (window) pool
constexpr uint32_t kInvalidRow = 0xFFFFFFFFu;    // padding or faulty key: zero row, no update
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

constexpr int kFlagFirst = 1;   // first chunk of its unit
constexpr int kFlagLast = 2;    // last chunk of its unit
constexpr int kFlagFinal = 4;   // last chunk of this CTA
constexpr int kFlagSetStart = 8;   // the chunk starts at the first key of its query's set

struct ChunkDesc {
  int32_t i;          // query token
  int32_t split;      // slice of the token's key set
  int32_t key_base;   // CSR position of the chunk's first key
  int32_t nkeys;      // keys in the chunk (tiles = ceil(nkeys / 64))
  int32_t flags;
  int32_t pad[3];
};

__device__ __forceinline__ int ceil_tiles(int nkeys) { return (nkeys + kT - 1) / kT; }

// Keys -> physical rows for one chunk. The chunk is shared by kParts
// resolver warps; part p's lanes handle keys p*kChunkKeys/kParts + lane,
// + lane + 32, ...; the loads of each phase are issued together so the
// chunk costs two round trips, not two per key. Prm holds the page tables
// and pool sizes.
// With inl_groups >= 0 the keys are not read from `indices` but built:
// position k of the set is group k below inl_groups (or group inl_list[k],
// a sorted list in shared memory, when inl_list is set) and window token
// inl_wstart + k - inl_groups after it (key_base is then the chunk's
// position in the set). inl_list may be this chunk's own table slot: every
// lane reads its keys before any lane writes a row.
template <int kParts = 1, class Prm>
__device__ void resolve_chunk(const Prm& P, int32_t b, int32_t key_base, int32_t nkeys, uint32_t* tab,
                              int lane, int part = 0, int32_t inl_groups = -1, int32_t inl_wstart = 0,
                              const int32_t* inl_list = nullptr) {
  constexpr int kPer = kChunkKeys / kParts / 32;
  const int k0 = part * (kChunkKeys / kParts);
  // Rows of lanes past the chunk's keys are skipped with a warp-uniform
  // branch, and faults are gathered into one status report at the end: a
  // short chunk (decode) then runs a few iterations of a short body, which
  // matters because the code is fetched cold on the first chunk of a launch.
  uint32_t err = 0;
  int32_t key[kPer];
#pragma unroll
  for (int e = 0; e < kPer; ++e) {
    key[e] = -2;
    if (k0 + 32 * e >= nkeys) continue;   // warp-uniform
    const int k = k0 + lane + 32 * e;
    const int32_t at = key_base + k;
    key[e] = k >= nkeys ? -2
             : inl_groups < 0 ? __ldg(P.indices + at)
             : at < inl_groups ? (inl_list != nullptr ? inl_list[at] : at)
             : (SPA_WINDOW_TAG | (inl_wstart + at - inl_groups));
  }
  __syncwarp();
  int32_t page[kPer];
#pragma unroll
  for (int e = 0; e < kPer; ++e) {
    page[e] = -1;
    if (k0 + 32 * e >= nkeys) continue;   // warp-uniform
    const int32_t kk = key[e];
    if (kk == -2) continue;
    if (kk < 0) { err |= SPA_DEV_BAD_INDEX; key[e] = -3; continue; }
    const bool raw = (kk & SPA_WINDOW_TAG) != 0;
    const int32_t t = kk & (SPA_WINDOW_TAG - 1);
    const int32_t* pt = raw ? P.pt_raw : P.pt_cmp;
    const int32_t cols = raw ? P.pt_raw_cols : P.pt_cmp_cols;
    const int32_t lp = t >> (raw ? P.raw_ps_log2 : P.cmp_ps_log2);
    if (pt == nullptr || lp >= cols) { err |= SPA_DEV_BAD_INDEX; key[e] = -3; continue; }
    page[e] = __ldg(pt + static_cast<int64_t>(b) * cols + lp);
  }
#pragma unroll
  for (int e = 0; e < kPer; ++e) {
    if (k0 + 32 * e >= nkeys) continue;   // warp-uniform
    const int k = k0 + lane + 32 * e;
    const int32_t kk = key[e];
    uint32_t row = kInvalidRow;
    if (kk >= 0) {
      const bool raw = (kk & SPA_WINDOW_TAG) != 0;
      const int32_t t = kk & (SPA_WINDOW_TAG - 1);
      const int32_t ps_log2 = raw ? P.raw_ps_log2 : P.cmp_ps_log2;
      const int64_t pages = raw ? P.raw_pages : P.cmp_pages;
      const int64_t pg = page[e];
      if (pg < 0 || pg >= pages) {
        err |= SPA_DEV_BAD_PAGE;
      } else {
        row = static_cast<uint32_t>((pg << ps_log2) + (t & ((1 << ps_log2) - 1))) | (raw ? kRawBit : 0u);
      }
    }
    if (k < nkeys) tab[k] = row;
  }
  if (err != 0) report(P.dev_status, err);
}

// ---- the complete groups a query's top-k row picks (sets built here)
// The row's entries j < width, loaded 16 per lane (entry 32 r + lane in
// register r, -1 past the width), become the ascending list of distinct
// groups g with 0 <= g < n_complete, written to `area` (kWords words of
// shared memory); returns the count.
constexpr int kInlineTopkMax = kInlineTopkMaxWidth;
constexpr int kTopkRegs = kInlineTopkMax / 32;
static_assert(kInlineTopkMax % 32 == 0, "whole registers per lane");
static_assert(kInlineTopkMax <= kChunkKeys, "the list of a unit fits its first chunk's table slot");

__device__ __forceinline__ void load_topk_row(const int32_t* row, int width, int lane, int32_t (&g)[kTopkRegs]) {
#pragma unroll
  for (int r = 0; r < kTopkRegs; ++r) g[r] = 32 * r + lane < width ? __ldg(row + 32 * r + lane) : -1;
}

// Through bitmaps rather than a sort (a sort of 512 entries costs about ten
// times the instructions, and the resolver shares its issue slots with a
// softmax warp). `area` holds the list in its first kInlineTopkMax words and
// a bitmap in the kWords - kInlineTopkMax after them: a window [w0, hi) of
// up to 32 * (kWords - kInlineTopkMax) groups gets one bit per group, every
// entry in the window sets its bit (repeats fall together), and the set
// bits' indices are appended to the list in ascending order, 32 words per
// step. The next window starts at the smallest entry not yet listed, so
// there are at most as many passes as windows holding an entry (one up to
// 4096 complete groups). The loops stay rolled: this code runs once per
// unit, and its size, not its speed, is what costs (the caller keeps it
// out of line for the same reason).
template <int kWords>
__device__ __forceinline__ int32_t pick_groups(const int32_t (&g)[kTopkRegs], int32_t n_complete, int lane,
                                               int32_t* area) {
  constexpr int kBitmapWords = kWords - kInlineTopkMax;
  static_assert(kBitmapWords >= 32 && kBitmapWords % 32 == 0, "room for a bitmap after the longest list");
  uint32_t* bits = reinterpret_cast<uint32_t*>(area + kInlineTopkMax);
  int32_t total = 0;
  int32_t w0 = 0;
  while (w0 < n_complete) {
    const int64_t span_end = w0 + 32LL * kBitmapWords;
    const int32_t hi = span_end < n_complete ? static_cast<int32_t>(span_end) : n_complete;
    const int words = (hi - w0 + 31) >> 5;
#pragma unroll 1
    for (int w = lane; w < words; w += 32) bits[w] = 0u;
    __syncwarp();
#pragma unroll
    for (int r = 0; r < kTopkRegs; ++r)
      if (g[r] >= w0 && g[r] < hi) atomicOr(bits + ((g[r] - w0) >> 5), 1u << ((g[r] - w0) & 31));
    __syncwarp();
#pragma unroll 1
    for (int b0 = 0; b0 < words; b0 += 32) {
      uint32_t m = b0 + lane < words ? bits[b0 + lane] : 0u;
      const int32_t c = __popc(m);
      int32_t incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int32_t t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      int32_t at = total + incl - c;
      const int32_t base = w0 + (b0 + lane) * 32;
#pragma unroll 1
      for (; m != 0u; m &= m - 1u) area[at++] = base + (__ffs(m) - 1);
      total += __shfl_sync(0xffffffffu, incl, 31);
    }
    __syncwarp();
    if (hi >= n_complete) break;
    int32_t nxt = INT_MAX;
#pragma unroll
    for (int r = 0; r < kTopkRegs; ++r)
      if (g[r] >= hi && g[r] < n_complete) nxt = min(nxt, g[r]);
    nxt = __reduce_min_sync(0xffffffffu, nxt);
    if (nxt == INT_MAX) break;
    w0 = nxt;
  }
  return total;
}

// A unit's picked groups, listed in the table slot `area` once the slot is
// free (its barrier `empty` at `parity`); the row's loads are in flight
// during the wait. Returns the count, or -1 when the wait gave up. Kept out
// of line: inlined into the resolver loop, the code grows the kernel enough
// to slow every launch of it, whether or not a launch takes this path.
static __device__ __noinline__ int32_t picked_groups_in_slot(const int32_t* row, int width, int32_t n_complete, int lane,
                                                             int32_t* area, uint64_t* empty, uint32_t parity,
                                                             volatile int* abort_flag, uint32_t* dev_status,
                                                             uint64_t wait_ns) {
  int32_t g[kTopkRegs];
  load_topk_row(row, width, lane, g);
  if (!mbar_wait(empty, parity, abort_flag, dev_status, wait_ns)) return -1;
  return pick_groups<kChunkKeys>(g, n_complete, lane, area);
}

// The resolver warp: walks this CTA's units (query i, slice), splits each
// slice's keys into chunks of up to kChunkKeys, resolves them into the
// double-buffered table and publishes a descriptor per chunk. An empty slice
// still gets one (empty) chunk so that every role sees every unit. S =
// slices per query. The CTA's units are every gridDim.x-th one (strided) or
// one contiguous range of about n_units / gridDim.x (contiguous: at any
// moment the CTAs then work on queries far apart, whose windows do not
// overlap). With kParts > 1, kParts warps run this loop side by side, each
// resolving its share of every chunk (tab_full then counts all of them);
// part 0 writes the descriptors.
// Sets built here from top-k rows: before a unit's first chunk the resolver
// waits for that chunk's table slot, builds the unit's sorted groups in it
// (the set's length depends on their count), and the chunk reads its keys
// from that list before its rows overwrite it. Every group position lies in
// the unit's first chunk (at most kInlineTopkMax <= kChunkKeys of them, at
// the front of the set).
template <int kParts = 1, class Prm>
__device__ void resolver_loop(const Prm& P, int S, uint32_t* tab, ChunkDesc* desc, uint64_t* tab_full,
                              uint64_t* tab_empty, volatile int* abort_flag, int lane, bool contiguous = false,
                              int part = 0) {
  int c = 0;
  const int64_t n_units = static_cast<int64_t>(P.n_queries) * S;
  const int64_t u0 = contiguous ? (static_cast<int64_t>(blockIdx.x) * n_units) / gridDim.x : blockIdx.x;
  const int64_t u_end = contiguous ? (static_cast<int64_t>(blockIdx.x + 1) * n_units) / gridDim.x : n_units;
  const int64_t step = contiguous ? 1 : gridDim.x;
  const bool picked = P.set_pos != nullptr && P.set_topk != nullptr && kParts == 1;
  for (int64_t u = u0; u < u_end && !*abort_flag; u += step) {
    const int i = static_cast<int>(u / S);
    const int split = static_cast<int>(u - static_cast<int64_t>(i) * S);
    int32_t set_begin = 0, set_len, inl_groups = -1, inl_wstart = 0;
    const int32_t b = __ldg(P.req + i);
    const bool b_ok = b >= 0 && b < P.n_requests;
    if (b_ok) {
      // The page-table rows of this request into L2 while the keys load,
      // so that the lookup after them (the third dependent load of the
      // chunk) hits L2: up to 64 lines (8 KB) of each table per lane group.
      const int32_t* rows[2] = {P.pt_raw + static_cast<int64_t>(b) * P.pt_raw_cols,
                                P.pt_cmp ? P.pt_cmp + static_cast<int64_t>(b) * P.pt_cmp_cols : nullptr};
      const int32_t cols[2] = {P.pt_raw_cols, P.pt_cmp ? P.pt_cmp_cols : 0};
#pragma unroll
      for (int tb = 0; tb < 2; ++tb) {
        const int lines = min(64, (cols[tb] + 31) / 32);
        for (int ln = lane; ln < lines; ln += 32) prefetch_l2(rows[tb] + 32 * ln);
      }
    }
    bool slot_held = false;   // the first chunk's slot is already waited for
    if (P.set_pos != nullptr) {
      // the set built here: the complete groups (all of them, or those the
      // top-k row picks, sorted, repeats removed), then the window
      const int32_t pos = __ldg(P.set_pos + i);
      const bool pos_ok = pos >= 0 && pos < SPA_WINDOW_TAG;
      const int32_t wn = pos_ok ? min(P.set_window, pos + 1) : 0;
      inl_groups = (pos_ok && P.set_ratio > 0) ? (pos + 1) / P.set_ratio : 0;
      if (picked) {
        inl_groups = picked_groups_in_slot(P.set_topk + static_cast<int64_t>(i) * P.set_topk_width,
                                           P.set_topk_width, inl_groups, lane,
                                           reinterpret_cast<int32_t*>(tab + (c & 1) * kChunkKeys),
                                           tab_empty + (c & 1), ((c >> 1) & 1) ^ 1, abort_flag, P.dev_status,
                                           P.wait_ns);
        if (inl_groups < 0) return;
        slot_held = true;
      }
      inl_wstart = pos + 1 - wn;
      set_len = pos_ok ? inl_groups + wn : -1;
    } else {
      set_begin = __ldg(P.indptr + i);
      set_len = __ldg(P.indptr + i + 1) - set_begin;
    }
    if (set_len < 0 || !b_ok) {
      if (lane == 0) report(P.dev_status, SPA_DEV_BAD_INDEX);
      set_len = 0;
    }
    const int tiles_total = ceil_tiles(set_len);
    const int tile_lo = static_cast<int>((static_cast<int64_t>(tiles_total) * split) / S);
    const int tile_hi = static_cast<int>((static_cast<int64_t>(tiles_total) * (split + 1)) / S);
    const int32_t key_lo = tile_lo * kT;
    const int32_t key_hi = min(tile_hi * kT, set_len);
    const bool final_unit = u + step >= u_end;
    int32_t k0 = key_lo;
    do {
      const int slot = c & 1;
      if (!slot_held && !mbar_wait(tab_empty + slot, ((c >> 1) & 1) ^ 1, abort_flag, P.dev_status, P.wait_ns))
        return;
      const int32_t n = max(0, min(kChunkKeys, key_hi - k0));   // 0: an empty slice
      resolve_chunk<kParts>(P, b, set_begin + k0, n, tab + slot * kChunkKeys, lane, part, inl_groups, inl_wstart,
                            slot_held ? reinterpret_cast<const int32_t*>(tab + slot * kChunkKeys) : nullptr);
      slot_held = false;
      if (lane == 0 && part == 0) {
        ChunkDesc& d = desc[slot];
        d.i = i;
        d.split = split;
        d.key_base = set_begin + k0;
        d.nkeys = n;
        const bool last = k0 + n >= key_hi;
        d.flags = (k0 == key_lo ? kFlagFirst : 0) | (last ? kFlagLast : 0) | (last && final_unit ? kFlagFinal : 0) |
                  (k0 == 0 && n > 0 ? kFlagSetStart : 0);
      }
      __syncwarp();
      mbar_arrive(tab_full + slot);
      ++c;
      k0 += n;
    } while (k0 < key_hi);
  }
}

// ------------------------------------------------------------------ host
inline int log2_exact(int32_t v) {
  int k = 0;
  while ((1 << k) < v) ++k;
  return k;
}

inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// A paged pool [rows, d] BF16 as a 2D tensor with a one-row, 64-column box,
// 128-byte swizzle: the form tile::gather4 takes.
inline bool encode_pool(CUtensorMap* m, const void* base, int64_t rows, int d) {
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(std::max<int64_t>(rows, 1))};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(d) * 2};
  const cuuint32_t box[2] = {64, 1};
  const cuuint32_t elem[2] = {1, 1};
  return tensor_map_encoder()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                              box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [N, H, d] BF16 with element strides (tok, head) as a 3D tensor {d, H, N},
// box {64, box_rows, 1}: one token's head rows, 64 columns at a time.
inline bool encode_q(CUtensorMap* m, const void* base, int32_t n, int32_t h, int d, int64_t stride_tok,
                     int64_t stride_head, int box_rows) {
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(h),
                              static_cast<cuuint64_t>(n)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(stride_head) * 2, static_cast<cuuint64_t>(stride_tok) * 2};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  const cuuint32_t elem[3] = {1, 1, 1};
  return tensor_map_encoder()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                              box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace attn
}  // namespace spa
