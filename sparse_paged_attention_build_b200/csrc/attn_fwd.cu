// Sparse paged attention with an attention sink, forward, on the sm_100a
// tensor cores (tcgen05 + TMEM).
//
// Page "Roadmap item 24 - joint compressed/window attention with sink",
// section "Reuse and arithmetic": compressed KV, the full recent window and
// the sink share one softmax denominator; the sink has no V; P and O are
// BF16 and LSE is the FP32 natural log of the denominator. Page "test: add
// block-level DeepSeek-V4 attention test", "What this test actually drives":
// the decode core runs over KV splits followed by a reduce, done here as an
// exact LSE merge.
//
// Work unit = (query token i, slice s of its key set, 128-head tile). All
// heads of the unit share every K/V row, so the unit is a dense MQA problem
// with M = 128 heads:
//   S  = Q[128 x d] . K_tile[64 x d]^T       tcgen05.mma, SMEM x SMEM -> TMEM
//   P  = exp2(S*scale*log2e - m)  (BF16)     softmax warps, TMEM -> regs -> TMEM
//   O += P[128 x 64] . V_tile[64 x d]         tcgen05.mma, TMEM x SMEM -> TMEM
// The sink seeds the running max and the denominator (m = sink*log2e,
// l = 1), so it is counted exactly once and never multiplies a V row.
//
// Warp roles (224 threads):
//   warps 0-3  softmax + epilogue; thread t owns head row t = TMEM lane t
//   warp  4    TMEM allocation; lane 0 issues every UMMA and commit
//   warps 5-6  paged gather: key -> page table -> 64-bit row address ->
//              16-byte cp.async of K and V rows into a 2-stage ring,
//              written in the 128-byte-swizzled K-major layout the UMMA
//              descriptors describe
// TMEM columns: S/P buffer 0 [0,64), buffer 1 [64,128), O [128,128+d).
// The running max is only moved when a tile's max exceeds it by more than
// 8 (log2 units), so P <= 256 and O is rescaled rarely; the final O/l and
// LSE use the same max, so the result is exact in exact arithmetic.
#include <cmath>

#include "spa_device.cuh"
#include "spa_internal.h"

namespace spa {
namespace {

constexpr int kT = kAttnKeysPerTile;   // keys per tile
constexpr int kStages = 2;
constexpr int kSoftThreads = 128;
constexpr int kMmaWarp = 4;
constexpr int kProdWarp0 = 5;
constexpr int kProdThreads = 64;
constexpr int kThreads = (kProdWarp0 * 32) + kProdThreads;   // 224
constexpr uint32_t kTmemCols = 256;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;

static_assert(kT == kProdThreads, "one producer thread resolves one key of a tile");

struct Params {
  const uint16_t* q;
  int64_t q_stride_tok, q_stride_head;
  int32_t n_queries, num_heads;
  const char* k_raw;
  const char* v_raw;
  int64_t raw_pages;
  int32_t raw_ps_log2, pt_raw_cols;
  const int32_t* pt_raw;
  const char* k_cmp;
  const char* v_cmp;
  int64_t cmp_pages;
  int32_t cmp_ps_log2, pt_cmp_cols;
  const int32_t* pt_cmp;
  const int32_t* req;
  int32_t n_requests;
  const int32_t* indptr;
  const int32_t* indices;
  const float* sink;
  float scale_log2;
  uint16_t* out;
  float* lse;
  int32_t num_splits;
  float* part_o;       // [n_queries * num_splits][num_heads][d]  (split runs only)
  float2* part_ml;     // [n_queries * num_splits][num_heads]
  uint32_t* tickets;   // [n_queries * head_tiles]
  uint32_t* dev_status;
};

template <int D>
struct Layout {
  static constexpr int kQBytes = 128 * D * 2;
  static constexpr int kTileBytes = kT * D * 2;             // one K or V tile
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kQOff = 0;
  static constexpr int kStageOff = kQBytes;
  static constexpr int kRowPtrOff = kStageOff + kStages * kStageBytes;   // [stages][T][2] ptrs
  static constexpr int kBarOff = kRowPtrOff + kStages * kT * 16;
  static constexpr int kNumBars = 1 + 2 * kStages + 2 + 2 + 2;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kUsed = kMiscOff + 16;
  // keep at most two CTAs per SM: TMEM holds two 256-column allocations
  static constexpr int kBytes = (kUsed + 1024) < 96 * 1024 ? 96 * 1024 : (kUsed + 1024);
  static constexpr uint32_t kOCol = 2 * kT;
  static_assert(kOCol + D <= kTmemCols, "TMEM budget");
  static_assert(kBytes * 2 <= 227 * 1024, "two CTAs per SM");
};

// Resolve one key to its K and V row pointers (nullptr for padding or a
// faulty key, which is zero-filled).
__device__ __forceinline__ void resolve_key(const Params& P, int32_t b, int32_t key, int row_bytes,
                                            const char*& kp, const char*& vp) {
  kp = nullptr;
  vp = nullptr;
  if (key < 0) {
    report(P.dev_status, SPA_DEV_BAD_INDEX);
    return;
  }
  const bool window = (key & SPA_WINDOW_TAG) != 0;
  const int32_t t = key & (SPA_WINDOW_TAG - 1);
  const int32_t* pt = window ? P.pt_raw : P.pt_cmp;
  const int32_t cols = window ? P.pt_raw_cols : P.pt_cmp_cols;
  const int32_t ps_log2 = window ? P.raw_ps_log2 : P.cmp_ps_log2;
  const int64_t pages = window ? P.raw_pages : P.cmp_pages;
  const int32_t lp = t >> ps_log2;
  if (pt == nullptr || lp >= cols) {
    report(P.dev_status, SPA_DEV_BAD_INDEX);
    return;
  }
  const int64_t page = pt[static_cast<int64_t>(b) * cols + lp];
  if (page < 0 || page >= pages) {
    report(P.dev_status, SPA_DEV_BAD_PAGE);
    return;
  }
  const int64_t row = (page << ps_log2) + (t & ((1 << ps_log2) - 1));
  const int64_t off = row * row_bytes;
  kp = (window ? P.k_raw : P.k_cmp) + off;
  vp = (window ? P.v_raw : P.v_cmp) + off;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 2) sparse_sink_attn_kernel(const Params P) {
  using L = Layout<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = bars + 1 + kStages;
  uint64_t* s_full = bars + 1 + 2 * kStages;
  uint64_t* p_ready = s_full + 2;
  uint64_t* o_done = p_ready + 2;
  uint64_t* mma_done = o_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);
  uint32_t* ticket_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff + 8);
  const char** rowptr = reinterpret_cast<const char**>(smem + L::kRowPtrOff);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int S = P.num_splits;
  const int i = blockIdx.x / S;
  const int split = blockIdx.x - i * S;
  const int head0 = blockIdx.y * 128;
  const int heads_here = min(128, P.num_heads - head0);

  // ---- the unit's key range
  int32_t set_begin = P.indptr[i];
  int32_t set_len = P.indptr[i + 1] - set_begin;
  const int32_t b = P.req[i];
  if (set_len < 0 || b < 0 || b >= P.n_requests) {
    if (tid == 0) report(P.dev_status, SPA_DEV_BAD_INDEX);
    set_len = 0;
  }
  const int tiles_total = (set_len + kT - 1) / kT;
  const int tile_lo = static_cast<int>((static_cast<int64_t>(tiles_total) * split) / S);
  const int tile_hi = static_cast<int>((static_cast<int64_t>(tiles_total) * (split + 1)) / S);
  const int ntiles = tile_hi - tile_lo;
  const int32_t key_lo = tile_lo * kT;
  const int32_t key_hi = min(tile_hi * kT, set_len);

  // ---- setup
  if (tid == 0) {
    mbar_init(q_full, kProdThreads);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(kv_full + s, kProdThreads);
      mbar_init(kv_empty + s, 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(s_full + s, 1);
      mbar_init(p_ready + s, kSoftThreads);
    }
    mbar_init(o_done, 1);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  if (warp >= kProdWarp0) {
    // ================================================= producers
    const int pt = tid - kProdWarp0 * 32;
    if (ntiles > 0) {
      // Q rows (zero rows past the unit's heads)
      const char* qbase = reinterpret_cast<const char*>(P.q);
      constexpr int kChunksPerRow = D / 8;   // 16-byte chunks
      for (int c = pt; c < 128 * kChunksPerRow; c += kProdThreads) {
        const int r = c / kChunksPerRow, ch = c % kChunksPerRow;
        const int db = ch >> 3, u = ch & 7;
        const uint32_t dst = sbase + L::kQOff + db * (128 * 128) + r * 128 + ((u ^ (r & 7)) << 4);
        const bool ok = r < heads_here;
        const char* src = ok ? qbase + 2 * (static_cast<int64_t>(i) * P.q_stride_tok +
                                            static_cast<int64_t>(head0 + r) * P.q_stride_head) + ch * 16
                             : qbase;
        cp_async16(dst, src, ok ? 16u : 0u);
      }
      cp_async_arrive_noinc(q_full);

      const char* dummy = P.k_raw;
      for (int jt = 0; jt < ntiles; ++jt) {
        const int stage = jt % kStages;
        if (!mbar_wait(kv_empty + stage, ((jt / kStages) & 1) ^ 1, abort_flag, P.dev_status)) break;
        // resolve this thread's key
        const int32_t kpos = key_lo + jt * kT + pt;
        const char* kp = nullptr;
        const char* vp = nullptr;
        if (kpos < key_hi) resolve_key(P, b, P.indices[set_begin + kpos], D * 2, kp, vp);
        rowptr[(stage * kT + pt) * 2 + 0] = kp;
        rowptr[(stage * kT + pt) * 2 + 1] = vp;
        named_bar_sync(1, kProdThreads);
        const uint32_t kdst = sbase + L::kStageOff + stage * L::kStageBytes;
        const uint32_t vdst = kdst + L::kTileBytes;
        for (int c = pt; c < kT * kChunksPerRow; c += kProdThreads) {
          const int r = c / kChunksPerRow, ch = c % kChunksPerRow;
          const int db = ch >> 3, u = ch & 7;
          const uint32_t off = db * (kT * 128) + r * 128 + ((u ^ (r & 7)) << 4);
          const char* ks = rowptr[(stage * kT + r) * 2 + 0];
          const char* vs = rowptr[(stage * kT + r) * 2 + 1];
          cp_async16(kdst + off, ks ? ks + ch * 16 : dummy, ks ? 16u : 0u);
          cp_async16(vdst + off, vs ? vs + ch * 16 : dummy, vs ? 16u : 0u);
        }
        cp_async_arrive_noinc(kv_full + stage);
      }
      cp_async_wait_all();
    }
  } else if (warp == kMmaWarp) {
    // ================================================= UMMA issuer
    if ((tid & 31) == 0 && ntiles > 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, kT, 0);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, D, 1);
      const uint32_t q_addr = sbase + L::kQOff;
      bool ok = mbar_wait(q_full, 0, abort_flag, P.dev_status);
      fence_proxy_async_smem();
      auto issue_pv = [&](int j) -> bool {
        const int sb = j & 1, st = j % kStages;
        if (!mbar_wait(p_ready + sb, (j >> 1) & 1, abort_flag, P.dev_status)) return false;
        tc_fence_after_sync();
        const uint32_t v_addr = sbase + L::kStageOff + st * L::kStageBytes + L::kTileBytes;
#pragma unroll
        for (int k = 0; k < kT / 16; ++k) {
          const uint64_t bdesc = smem_desc_sw128(v_addr + k * 16 * 128, kT * 128, 1024);
          umma_ts(tmem + L::kOCol, tmem + sb * kT + k * 8, bdesc, idesc_o,
                  (j > 0 || k > 0) ? 1u : 0u);
        }
        tc_commit(kv_empty + st);
        tc_commit(o_done);
        return true;
      };
      for (int jt = 0; ok && jt < ntiles; ++jt) {
        const int stage = jt % kStages, sb = jt & 1;
        if (!mbar_wait(kv_full + stage, (jt / kStages) & 1, abort_flag, P.dev_status)) { ok = false; break; }
        fence_proxy_async_smem();
        tc_fence_after_sync();
        const uint32_t k_addr = sbase + L::kStageOff + stage * L::kStageBytes;
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t koff = (k & 3) * 32;   // 16 elements = 32 bytes inside the swizzle atom
          const uint64_t adesc = smem_desc_sw128(q_addr + (k >> 2) * (128 * 128) + koff, 16, 1024);
          const uint64_t bdesc = smem_desc_sw128(k_addr + (k >> 2) * (kT * 128) + koff, 16, 1024);
          umma_ss(tmem + sb * kT, adesc, bdesc, idesc_s, k > 0 ? 1u : 0u);
        }
        tc_commit(s_full + sb);
        if (jt >= 1 && !issue_pv(jt - 1)) { ok = false; break; }
      }
      if (ok) ok = issue_pv(ntiles - 1);
      // every UMMA has completed before TMEM is released
      tc_commit(mma_done);
      mbar_wait(mma_done, 0, nullptr, P.dev_status);
    }
  } else {
    // ================================================= softmax + epilogue
    const int row = tid;   // head row == TMEM lane
    const int h = head0 + row;
    const bool row_ok = row < heads_here;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    float m = -INFINITY, l = 0.f;
    if (split == 0 && P.sink != nullptr && row_ok) {
      m = P.sink[h] * kLog2e;
      l = 1.f;
      if (!(m > -INFINITY)) { m = -INFINITY; l = 0.f; }
    }
    bool ok = true;
    for (int jt = 0; jt < ntiles; ++jt) {
      const int sb = jt & 1;
      // tcgen05.ld/st are warp-collective: keep every branch warp-uniform
      if (!__all_sync(0xffffffffu, mbar_wait(s_full + sb, (jt >> 1) & 1, abort_flag, P.dev_status))) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
      const int nv = min(kT, key_hi - (key_lo + jt * kT));
      uint32_t s0[32], s1[32];
      tmem_ld32(lane_addr + sb * kT, s0);
      tmem_ld32(lane_addr + sb * kT + 32, s1);
      tmem_ld_wait(s0);
      tmem_ld_wait(s1);
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        if (c < nv) mx = fmaxf(mx, __uint_as_float(s0[c]));
        if (c + 32 < nv) mx = fmaxf(mx, __uint_as_float(s1[c]));
      }
      const float tmax = mx * P.scale_log2;
      const bool move = tmax > m + kRescaleThreshold || (m == -INFINITY && tmax > -INFINITY);
      const float alpha = !move ? 1.f : (m == -INFINITY ? 0.f : exp2_approx(m - tmax));
      l *= alpha;
      if (move) m = tmax;
      if (jt > 0 && __any_sync(0xffffffffu, move)) {
        // rows whose max moved rescale their O row (alpha = 1 elsewhere);
        // PV(jt-1) must have landed in TMEM first
        if (!__all_sync(0xffffffffu, mbar_wait(o_done, (jt - 1) & 1, abort_flag, P.dev_status))) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t o[32];
          tmem_ld32(lane_addr + L::kOCol + c0, o);
          tmem_ld_wait(o);
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
          tmem_st32(lane_addr + L::kOCol + c0, o);
        }
        tmem_st_wait();
      }
      const float neg_m = -m;
      float sum = 0.f;
      uint32_t pk[32];
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const float p0 = (2 * c < nv) ? exp2_approx(fmaf(__uint_as_float(s0[2 * c]), P.scale_log2, neg_m)) : 0.f;
        const float p1 = (2 * c + 1 < nv) ? exp2_approx(fmaf(__uint_as_float(s0[2 * c + 1]), P.scale_log2, neg_m)) : 0.f;
        const float p2 = (2 * c + 32 < nv) ? exp2_approx(fmaf(__uint_as_float(s1[2 * c]), P.scale_log2, neg_m)) : 0.f;
        const float p3 = (2 * c + 33 < nv) ? exp2_approx(fmaf(__uint_as_float(s1[2 * c + 1]), P.scale_log2, neg_m)) : 0.f;
        sum += (p0 + p1) + (p2 + p3);
        pk[c] = pack_bf16x2(p0, p1);
        pk[c + 16] = pack_bf16x2(p2, p3);
      }
      l += sum;
      tmem_st32(lane_addr + sb * kT, pk);   // P overwrites the first 32 columns of S
      tmem_st_wait();
      tc_fence_before_sync();
      mbar_arrive(p_ready + sb);
    }
    if (ok && ntiles > 0) {
      ok = __all_sync(0xffffffffu, mbar_wait(o_done, (ntiles - 1) & 1, abort_flag, P.dev_status));
      tc_fence_after_sync();
    }
    const bool have_o = ok && ntiles > 0;
    if (S == 1) {
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
      uint16_t* orow = P.out + (static_cast<int64_t>(i) * P.num_heads + h) * D;
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t o[32];
        if (have_o) {
          tmem_ld32(lane_addr + L::kOCol + c0, o);
          tmem_ld_wait(o);
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = 0u;
        }
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 16; ++c)
          pk[c] = pack_bf16x2(__uint_as_float(o[2 * c]) * inv_l, __uint_as_float(o[2 * c + 1]) * inv_l);
        if (row_ok) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
          for (int v = 0; v < 4; ++v) dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
        }
      }
      if (row_ok) P.lse[static_cast<int64_t>(i) * P.num_heads + h] = l > 0.f ? (m + log2_approx(l)) * kLn2 : -INFINITY;
    } else {
      // partial result of this slice (no normalisation), then the last
      // slice to finish merges all of them
      const int64_t unit = static_cast<int64_t>(i) * S + split;
      float* prow = P.part_o + (unit * P.num_heads + h) * D;
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t o[32];
        if (have_o) {
          tmem_ld32(lane_addr + L::kOCol + c0, o);
          tmem_ld_wait(o);
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = 0u;
        }
        if (row_ok) {
          float4* dst = reinterpret_cast<float4*>(prow + c0);
#pragma unroll
          for (int v = 0; v < 8; ++v)
            dst[v] = make_float4(__uint_as_float(o[4 * v]), __uint_as_float(o[4 * v + 1]),
                                 __uint_as_float(o[4 * v + 2]), __uint_as_float(o[4 * v + 3]));
        }
      }
      if (row_ok) P.part_ml[unit * P.num_heads + h] = make_float2(m, l);
      __threadfence();
      named_bar_sync(2, kSoftThreads);
      if (tid == 0) *ticket_slot = atomicAdd(P.tickets + static_cast<int64_t>(i) * gridDim.y + blockIdx.y, 1u);
      named_bar_sync(2, kSoftThreads);
      if (*ticket_slot == static_cast<uint32_t>(S - 1) && row_ok) {
        __threadfence();
        float M = -INFINITY;
        for (int s = 0; s < S; ++s) {
          const float2 ml = __ldcg(P.part_ml + (static_cast<int64_t>(i) * S + s) * P.num_heads + h);
          if (ml.y > 0.f) M = fmaxf(M, ml.x);
        }
        float Lsum = 0.f;
        float w[kAttnMaxSplits];
#pragma unroll
        for (int s = 0; s < kAttnMaxSplits; ++s) {
          w[s] = 0.f;
          if (s < S) {
            const float2 ml = __ldcg(P.part_ml + (static_cast<int64_t>(i) * S + s) * P.num_heads + h);
            w[s] = (ml.y > 0.f) ? exp2_approx(ml.x - M) : 0.f;
            Lsum += w[s] * ml.y;
          }
        }
        const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
        uint16_t* orow = P.out + (static_cast<int64_t>(i) * P.num_heads + h) * D;
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 8) {
          float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
          for (int s = 0; s < S; ++s) {
            if (w[s] == 0.f) continue;
            const float4* src = reinterpret_cast<const float4*>(
                P.part_o + (((static_cast<int64_t>(i) * S + s) * P.num_heads + h) * D + c0));
            const float4 a = __ldcg(src), bq = __ldcg(src + 1);
            acc[0] += w[s] * a.x; acc[1] += w[s] * a.y; acc[2] += w[s] * a.z; acc[3] += w[s] * a.w;
            acc[4] += w[s] * bq.x; acc[5] += w[s] * bq.y; acc[6] += w[s] * bq.z; acc[7] += w[s] * bq.w;
          }
          *reinterpret_cast<uint4*>(orow + c0) =
              make_uint4(pack_bf16x2(acc[0] * inv, acc[1] * inv), pack_bf16x2(acc[2] * inv, acc[3] * inv),
                         pack_bf16x2(acc[4] * inv, acc[5] * inv), pack_bf16x2(acc[6] * inv, acc[7] * inv));
        }
        P.lse[static_cast<int64_t>(i) * P.num_heads + h] = Lsum > 0.f ? (M + log2_approx(Lsum)) * kLn2 : -INFINITY;
      }
    }
  }

  // ---- teardown: every TMEM access above has completed
  __syncwarp();
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

template <int D>
cudaError_t launch_d(const Params& P, int head_tiles, cudaStream_t stream) {
  using L = Layout<D>;
  static bool configured = false;
  if (!configured) {
    cudaError_t err = cudaFuncSetAttribute(sparse_sink_attn_kernel<D>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes);
    if (err != cudaSuccess) return err;
    configured = true;
  }
  dim3 grid(static_cast<unsigned>(P.n_queries) * P.num_splits, head_tiles);
  sparse_sink_attn_kernel<D><<<grid, kThreads, L::kBytes, stream>>>(P);
  return cudaGetLastError();
}

int log2_exact(int32_t v) {
  int k = 0;
  while ((1 << k) < v) ++k;
  return k;
}

}  // namespace

size_t attn_workspace_bytes(int32_t n_queries, int32_t num_heads, int32_t head_dim,
                            int32_t num_splits) {
  if (num_splits <= 1) return 0;
  const int64_t units = static_cast<int64_t>(n_queries) * num_splits;
  const int64_t head_tiles = (num_heads + 127) / 128;
  size_t bytes = static_cast<size_t>(units * num_heads * head_dim) * sizeof(float);   // part_o
  bytes += static_cast<size_t>(units * num_heads) * sizeof(float2);                   // part_ml
  bytes += static_cast<size_t>(n_queries * head_tiles) * sizeof(uint32_t);            // tickets
  return bytes + 256;
}

cudaError_t launch_sparse_sink_attn(const AttnArgs& a, cudaStream_t stream) {
  if (a.n_queries == 0) return cudaSuccess;
  Params P;
  P.q = a.q;
  P.q_stride_tok = a.q_stride_tok;
  P.q_stride_head = a.q_stride_head;
  P.n_queries = a.n_queries;
  P.num_heads = a.num_heads;
  P.k_raw = reinterpret_cast<const char*>(a.k_raw);
  P.v_raw = reinterpret_cast<const char*>(a.v_raw);
  P.raw_pages = a.raw_num_pages;
  P.raw_ps_log2 = log2_exact(a.raw_page_size);
  P.pt_raw = a.pt_raw;
  P.pt_raw_cols = a.pt_raw_cols;
  P.k_cmp = reinterpret_cast<const char*>(a.k_cmp);
  P.v_cmp = reinterpret_cast<const char*>(a.v_cmp);
  P.cmp_pages = a.pt_cmp ? a.cmp_num_pages : 0;
  P.cmp_ps_log2 = a.pt_cmp ? log2_exact(a.cmp_page_size) : 0;
  P.pt_cmp = a.pt_cmp;
  P.pt_cmp_cols = a.pt_cmp ? a.pt_cmp_cols : 0;
  P.req = a.req;
  P.n_requests = a.n_requests;
  P.indptr = a.indptr;
  P.indices = a.indices;
  P.sink = a.sink;
  P.scale_log2 = static_cast<float>(static_cast<double>(a.scale) * 1.4426950408889634);
  P.out = a.out;
  P.lse = a.lse;
  P.num_splits = a.num_splits;
  P.dev_status = a.dev_status;
  const int head_tiles = (a.num_heads + 127) / 128;
  P.part_o = nullptr;
  P.part_ml = nullptr;
  P.tickets = nullptr;
  if (a.num_splits > 1) {
    const int64_t units = static_cast<int64_t>(a.n_queries) * a.num_splits;
    char* ws = static_cast<char*>(a.workspace);
    P.part_o = reinterpret_cast<float*>(ws);
    ws += units * a.num_heads * a.head_dim * sizeof(float);
    P.part_ml = reinterpret_cast<float2*>(ws);
    ws += units * a.num_heads * sizeof(float2);
    P.tickets = reinterpret_cast<uint32_t*>(ws);
    cudaError_t err = cudaMemsetAsync(P.tickets, 0,
                                      static_cast<size_t>(a.n_queries) * head_tiles * sizeof(uint32_t), stream);
    if (err != cudaSuccess) return err;
  }
  return a.head_dim == 128 ? launch_d<128>(P, head_tiles, stream) : launch_d<64>(P, head_tiles, stream);
}

}  // namespace spa
