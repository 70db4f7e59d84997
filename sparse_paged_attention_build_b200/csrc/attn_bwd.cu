// Backward of the sparse paged attention with an attention sink, on the
// sm_100a tensor cores (tcgen05 + TMEM).
//
// Page "Roadmap item 24 - joint compressed/window attention with sink"
// names the backward as its follow-on item: dQ, dK/dV scattered to the
// pages, and d_sink, from the saved O and LSE. For one (query i, head h)
// over the keys j of its set, with the probabilities recomputed from the
// saved LSE (natural log, sink included):
//   p_j = exp(scale q.k_j - LSE),  D = dO . O,  dp_j = dO . v_j,
//   ds_j = p_j (dp_j - D),  dq = scale sum_j ds_j k_j,
//   dk_j += scale ds_j q,  dv_j += p_j dO,  dsink_h += -exp(sink_h - LSE) D
// (the sink's logit has no V, so its dp is 0).
//
// Work unit = (query token, key slice, 128-head tile), as in the forward.
// All heads share every K/V row, so each 64-key tile is five dense products:
//   S    = Q  . K^T   [128 heads x 64 keys], K-dim d       -> TMEM
//   dP   = dO . V^T   [128 heads x 64 keys], K-dim d       -> TMEM
//   dQ  += dS . K     [128 heads x d],       K-dim 64 keys -> TMEM, over the unit
//   dV^T = dO^T . P   [d x 64 keys],         K-dim 128 heads
//   dK^T = Q^T . dS   [d x 64 keys],         K-dim 128 heads
// The last two read the same shared-memory copies of Q and dO as M-major A
// operands and P/dS as N-major B operands, so the sum over heads of dk and
// dv happens inside the product: each tile leaves one d x 64 block per pool,
// added (FP32 reductions) into the gradient rows of the tile's keys.
//
// Persistent CTAs, one per SM (the shared-memory footprint and the
// 512-column TMEM allocation both say so). Warp roles (384 threads):
//   warps 0-3   thread t owns head row t (TMEM lane t): D = dO . O at the
//               start of a unit, then per tile P and dS from S, dP and the
//               saved LSE into shared memory (BF16, 128-byte swizzled)
//   warp  4     TMEM allocation; lane 0 issues every UMMA and commit
//   warp  5     resolver: keys -> physical rows (shared with the forward)
//   warp  6     K gather (TMA tile::gather4, 3-stage ring) and each unit's
//               Q and dO (TMA boxes)
//   warp  7     V gather (2-stage ring)
//   warps 8-11  thread t owns TMEM lane t: writes dV^T, then dK^T (d index
//               t) into a [key][d] FP32 staging tile whose rows the TMA adds
//               into the gradient pools (one bulk reduction per key), and at
//               the end of a unit reads dQ (head row t) and adds it into dq
// TMEM columns: two S|dP buffers [0,128) and [128,256), dV^T|dK^T
// [256,384), dQ [384,512). Per tile the UMMA thread issues S/dP of tile g
// (into buffer g&1, without waiting for the softmax of tile g-1) and then
// the dQ/dV/dK products of tile g-1 once its P and dS are written, so the
// softmax of consecutive tiles runs back to back while the tensor core does
// the rest.
#include <cmath>
#include <cstring>

#include "attn_common.cuh"

namespace spa {
namespace {

using namespace attn;

constexpr int kStagesK = 3;          // K is read by S (tile g) and by dQ (tile g, issued later)
constexpr int kStagesV = 2;
constexpr int kSoftThreads = 128;
constexpr int kMmaWarp = 4;
constexpr int kResolverWarp = 5;
constexpr int kKWarp = 6;
constexpr int kVWarp = 7;
constexpr int kRedWarp0 = 8;
constexpr int kThreads = 384;
constexpr uint32_t kTmemCols = 512;
// consumers of a chunk descriptor: K warp, V warp, MMA thread, softmax, reducers
constexpr uint32_t kTabConsumers = 32 + 32 + 1 + kSoftThreads + 128;

struct Params {
  CUtensorMap tm_q;       // 3D {d, H, N}, box {64, q_box_rows, 1}
  CUtensorMap tm_do;      // dO, same form
  CUtensorMap tm_k_raw;   // 2D {d, rows}, box {64, 1}: gather4 / single rows
  CUtensorMap tm_v_raw;
  CUtensorMap tm_k_cmp;
  CUtensorMap tm_v_cmp;
  int32_t q_box_rows;     // min(128, num_heads)
  int32_t n_queries, num_heads;
  int64_t raw_pages;
  int32_t raw_ps_log2, pt_raw_cols;
  const int32_t* pt_raw;
  int64_t cmp_pages;
  int32_t cmp_ps_log2, pt_cmp_cols;
  const int32_t* pt_cmp;
  const int32_t* req;
  int32_t n_requests;
  const int32_t* indptr;
  const int32_t* indices;
  // non-NULL: the sets are built in the resolver from the positions (the
  // complete ratio-set_ratio groups -- all of them, or those the set_topk
  // row picks, sorted -- then the window of set_window tokens) instead of
  // read from indptr/indices
  const int32_t* set_pos;
  int32_t set_window, set_ratio;
  const int32_t* set_topk;   // [n_queries, set_topk_width] or NULL
  int32_t set_topk_width;
  const float* sink;
  float scale, scale_log2;
  const uint16_t* o;      // saved O [N, H, d]
  const float* lse;       // saved LSE [N, H]
  float* dq;              // [N, H, d]
  float* dk_raw;          // [raw rows, d]
  float* dv_raw;
  float* dk_cmp;          // [cmp rows, d]
  float* dv_cmp;
  float* dsink;           // [H] or NULL
  int32_t num_splits;
  uint32_t* dev_status;
  uint64_t wait_ns;   // limit of the waits between the roles
};

template <int D>
struct Layout {
  static constexpr int kHalfBytes = 128 * 128;                  // [128 rows][64 cols] BF16
  static constexpr int kTileBytes = kT * D * 2;                 // one K or V tile
  static constexpr int kPBytes = 128 * kT * 2;                  // one P or dS tile [128 heads][64 keys]
  static constexpr int kQOff = 0;                               // Q  [2 halves]
  static constexpr int kDOOff = 2 * kHalfBytes;                 // dO [2 halves]
  static constexpr int kKOff = 4 * kHalfBytes;
  static constexpr int kVOff = kKOff + kStagesK * kTileBytes;
  static constexpr int kPOff = kVOff + kStagesV * kTileBytes;   // P, then dS
  static constexpr int kBulkOff = kPOff + 2 * kPBytes;          // [64 keys][D] FP32: a dV or dK tile
  static constexpr int kTabOff = kBulkOff + kT * D * 4;         // [2][kChunkKeys] u32
  static constexpr int kDescOff = kTabOff + 2 * kChunkKeys * 4;
  static constexpr int kBarOff = kDescOff + 2 * static_cast<int>(sizeof(ChunkDesc));
  // tab_full[2], tab_empty[2], qd_full, qd_empty, K ring, V ring, s_full[2],
  // p_ready, pd_free, g_full, g_free, dq_full, dq_free, mma_done, red_sync[2]
  static constexpr int kNumBars = 2 + 2 + 2 + 2 * kStagesK + 2 * kStagesV + 2 + 1 + 1 + 1 + 1 + 3 + 2;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  // a 2 KB staging area per reducer warp: gradient rows leave through it as
  // coalesced 16-byte reductions
  static constexpr int kStageOff = (kMiscOff + 16 + 127) / 128 * 128;
  static constexpr int kUsed = kStageOff + 4 * 2048;
  static constexpr int kBytes = kUsed + 1024;                   // + alignment slack
  static constexpr uint32_t kSCol = 0;                          // buffer b: S at 128 b, dP at 128 b + 64
  static constexpr uint32_t kDPCol = kT;
  static constexpr uint32_t kGCol = 4 * kT;                     // dV^T, then dK^T
  static constexpr uint32_t kDQCol = kGCol + 2 * kT;
  static_assert(kDQCol + 128 <= kTmemCols, "TMEM budget");
  static_assert(kBytes <= 227 * 1024, "shared memory");
  static_assert(kPOff % 1024 == 0 && kKOff % 1024 == 0 && kVOff % 1024 == 0, "swizzle atoms");
  static_assert(kStageOff % 16 == 0, "16-byte staging accesses");
};

struct Bars {
  uint64_t* tab_full;   // [2]
  uint64_t* tab_empty;  // [2]
  uint64_t* qd_full;    // Q and dO of the unit landed
  uint64_t* qd_empty;   // every product reading them has completed
  uint64_t* k_full;     // [kStagesK]
  uint64_t* k_empty;
  uint64_t* v_full;     // [kStagesV]
  uint64_t* v_empty;
  uint64_t* s_full;     // [2] S and dP of buffer b in TMEM
  uint64_t* p_ready;    // P and dS of the current tile in shared memory (S/dP read)
  uint64_t* pd_free;    // the products reading P/dS have completed
  uint64_t* g_full;     // dV^T/dK^T of the tile complete
  uint64_t* g_free;     // ... and read out
  uint64_t* dq_full;    // dQ of the unit complete
  uint64_t* dq_free;    // ... and read out
  uint64_t* mma_done;
  // [2]: barrier of the reducer threads, the two used in turn (bounded)
  uint64_t* red_sync;
};

// 8 BF16 in a 16-byte word, times 8 BF16 in another, summed in FP32.
__device__ __forceinline__ float dot8_bf16(const uint4 a, const uint4 b) {
  const uint32_t wa[4] = {a.x, a.y, a.z, a.w};
  const uint32_t wb[4] = {b.x, b.y, b.z, b.w};
  float acc = 0.f;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float2 fa = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wa[k]));
    const float2 fb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wb[k]));
    acc = fmaf(fa.x, fb.x, acc);
    acc = fmaf(fa.y, fb.y, acc);
  }
  return acc;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1) sparse_sink_attn_bwd_kernel(const __grid_constant__ Params P) {
  using L = Layout<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bar0 = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  Bars B;
  B.tab_full = bar0;
  B.tab_empty = bar0 + 2;
  B.qd_full = bar0 + 4;
  B.qd_empty = bar0 + 5;
  B.k_full = bar0 + 6;
  B.k_empty = B.k_full + kStagesK;
  B.v_full = B.k_empty + kStagesK;
  B.v_empty = B.v_full + kStagesV;
  B.s_full = B.v_empty + kStagesV;
  B.p_ready = B.s_full + 2;
  B.pd_free = B.p_ready + 1;
  B.g_full = B.pd_free + 1;
  B.g_free = B.g_full + 1;
  B.dq_full = B.g_free + 1;
  B.dq_free = B.dq_full + 1;
  B.mma_done = B.dq_free + 1;
  B.red_sync = B.mma_done + 1;
  uint32_t* tab = reinterpret_cast<uint32_t*>(smem + L::kTabOff);
  ChunkDesc* desc = reinterpret_cast<ChunkDesc*>(smem + L::kDescOff);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int S = P.num_splits;
  const int head0 = blockIdx.y * 128;
  const int heads_here = min(128, P.num_heads - head0);

  // ---- setup. Q and dO rows the TMA never writes (heads past the tensor
  // when it has fewer than 128, the upper 64 columns when d = 64) must read
  // as zeros: the head-sum products run over all 128 rows and 128 columns.
  {
    uint4* z = reinterpret_cast<uint4*>(smem + L::kQOff);
    for (int k = tid; k < (4 * L::kHalfBytes) / 16; k += kThreads) z[k] = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
  }
  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(B.tab_full + s, 32);
      mbar_init(B.tab_empty + s, kTabConsumers);
      mbar_init(B.s_full + s, 1);
      mbar_init(B.red_sync + s, 128);
    }
    mbar_init(B.qd_full, 1);
    mbar_init(B.qd_empty, 1);
    for (int s = 0; s < kStagesK; ++s) {
      mbar_init(B.k_full + s, 1);
      mbar_init(B.k_empty + s, 1);
    }
    for (int s = 0; s < kStagesV; ++s) {
      mbar_init(B.v_full + s, 1);
      mbar_init(B.v_empty + s, 1);
    }
    mbar_init(B.pd_free, 1);
    mbar_init(B.g_full, 1);
    mbar_init(B.g_free, 128);
    mbar_init(B.p_ready, kSoftThreads);
    mbar_init(B.dq_full, 1);
    mbar_init(B.dq_free, 128);
    mbar_init(B.mma_done, 1);
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

  if (warp == kResolverWarp) {
    // ================================================= resolver
    // contiguous ranges of units: concurrent CTAs then add into distant
    // gradient rows (consecutive queries share most of their window keys)
    resolver_loop(P, S, tab, desc, B.tab_full, B.tab_empty, abort_flag, lane, true);
  } else if (warp == kKWarp || warp == kVWarp) {
    // ================================================= K / V gather (TMA)
    // As in the forward: lane j issues one tile::gather4 (four rows, 64
    // columns) per job; rows past the chunk and faulty keys are zero-filled.
    // Lane 0 of the K warp also loads Q and dO of every unit that has keys.
    const bool is_k = warp == kKWarp;
    const int nst = is_k ? kStagesK : kStagesV;
    uint64_t* full = is_k ? B.k_full : B.v_full;
    uint64_t* empty = is_k ? B.k_empty : B.v_empty;
    const CUtensorMap* map_raw = is_k ? &P.tm_k_raw : &P.tm_v_raw;
    const CUtensorMap* map_cmp = is_k ? &P.tm_k_cmp : &P.tm_v_cmp;
    const uint32_t ring = sbase + (is_k ? L::kKOff : L::kVOff);
    constexpr int kHalves = D / 64;
    constexpr int kGroups = kT / 4;
    constexpr int kJobs = kGroups * kHalves;
    const int grp = lane % kGroups, half = lane / kGroups;
    const bool issuer = lane < kJobs;
    int c = 0, g = 0, qc = 0;
    bool final_seen = false;
    while (!final_seen) {
      const int slot = c & 1;
      if (!mbar_wait(B.tab_full + slot, (c >> 1) & 1, abort_flag, P.dev_status)) break;
      const ChunkDesc d = desc[slot];
      final_seen = (d.flags & kFlagFinal) != 0;
      const uint32_t* t_rows = tab + slot * kChunkKeys;
      const int ntiles = ceil_tiles(d.nkeys);
      bool ok = true;
      if (is_k && (d.flags & kFlagFirst) && ntiles > 0) {
        ok = mbar_wait(B.qd_empty, (qc & 1) ^ 1, abort_flag, P.dev_status);
        if (ok && lane == 0) {
          mbar_arrive_expect_tx(B.qd_full, 2 * P.q_box_rows * 128 * kHalves);
          for (int hb = 0; hb < kHalves; ++hb) {
            tma_load_3d(sbase + L::kQOff + hb * L::kHalfBytes, &P.tm_q, B.qd_full, hb * 64, head0, d.i);
            tma_load_3d(sbase + L::kDOOff + hb * L::kHalfBytes, &P.tm_do, B.qd_full, hb * 64, head0, d.i);
          }
        }
        ++qc;
      }
      for (int t = 0; ok && t < ntiles; ++t, ++g) {
        const int stage = g % nst;
        if (!mbar_wait(empty + stage, ((g / nst) & 1) ^ 1, abort_flag, P.dev_status)) { ok = false; break; }
        if (lane == 0) mbar_arrive_expect_tx(full + stage, L::kTileBytes);
        __syncwarp();
        if (issuer) {
          const int nv = min(kT, d.nkeys - t * kT);
          uint32_t e[4];
          bool any_raw = false, any_cmp = false;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int r = 4 * grp + k;
            e[k] = r < nv ? t_rows[t * kT + r] : kInvalidRow;
            if (e[k] != kInvalidRow) {
              if (e[k] & kRawBit) any_raw = true;
              else any_cmp = true;
            }
          }
          int32_t y[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) y[k] = e[k] == kInvalidRow ? -1 : static_cast<int32_t>(e[k] & ~kRawBit);
          const uint32_t dst = ring + stage * L::kTileBytes + half * (kT * 128) + (4 * grp) * 128;
          if (!(any_raw && any_cmp)) {
            tma_gather4(dst, any_cmp ? map_cmp : map_raw, full + stage, half * 64, y[0], y[1], y[2], y[3]);
          } else {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const bool cmp_row = e[k] != kInvalidRow && !(e[k] & kRawBit);
              tma_load_2d(dst + k * 128, cmp_row ? map_cmp : map_raw, full + stage, half * 64, y[k]);
            }
          }
        }
      }
      mbar_arrive(B.tab_empty + slot);
      ++c;
      if (!ok) break;
    }
  } else if (warp == kMmaWarp) {
    // ================================================= UMMA issuer
    if (lane == 0) {
      constexpr uint32_t id_s = idesc_bf16_f32_ab(128, kT, 0, 0);   // S, dP
      constexpr uint32_t id_dq = idesc_bf16_f32_ab(128, D, 0, 1);   // dQ += dS K
      constexpr uint32_t id_g = idesc_bf16_f32_ab(128, kT, 1, 1);   // dV^T, dK^T
      const uint32_t q_addr = sbase + L::kQOff, do_addr = sbase + L::kDOOff;
      int c = 0, g = 0, u = 0, ud = 0;
      bool ok = true, final_seen = false;
      bool pending = false, p_first = false, p_last = false;
      int pg = 0;
      // dQ, dV^T and dK^T of tile gg (its P and dS are in shared memory)
      auto issue_d = [&](int gg, bool first, bool last) -> bool {
        if (!mbar_wait(B.g_free, (gg & 1) ^ 1, abort_flag, P.dev_status)) return false;
        if (first) {
          if (!mbar_wait(B.dq_free, (ud & 1) ^ 1, abort_flag, P.dev_status)) return false;
          ++ud;
        }
        tc_fence_after_sync();
        const uint32_t k_addr = sbase + L::kKOff + (gg % kStagesK) * L::kTileBytes;
        const uint32_t p_addr = sbase + L::kPOff;
        const uint32_t ds_addr = p_addr + L::kPBytes;
        const uint32_t gcol = L::kGCol;
#pragma unroll
        for (int k = 0; k < kT / 16; ++k) {   // K-dim: 16 keys per step
          const uint64_t a = smem_desc_sw128(ds_addr + k * 32, 16, 1024);
          const uint64_t b = smem_desc_sw128(k_addr + k * 16 * 128, kT * 128, 1024);
          umma_ss(tmem + L::kDQCol, a, b, id_dq, (!first || k > 0) ? 1u : 0u);
        }
#pragma unroll
        for (int k = 0; k < 128 / 16; ++k) {  // K-dim: 16 heads per step
          const uint64_t a = smem_desc_sw128(do_addr + k * 16 * 128, L::kHalfBytes, 1024);
          const uint64_t b = smem_desc_sw128(p_addr + k * 16 * 128, L::kPBytes, 1024);
          umma_ss(tmem + gcol, a, b, id_g, k > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int k = 0; k < 128 / 16; ++k) {
          const uint64_t a = smem_desc_sw128(q_addr + k * 16 * 128, L::kHalfBytes, 1024);
          const uint64_t b = smem_desc_sw128(ds_addr + k * 16 * 128, L::kPBytes, 1024);
          umma_ss(tmem + gcol + kT, a, b, id_g, k > 0 ? 1u : 0u);
        }
        tc_commit(B.k_empty + gg % kStagesK);
        tc_commit(B.pd_free);
        tc_commit(B.g_full);
        if (last) {
          tc_commit(B.dq_full);
          tc_commit(B.qd_empty);
        }
        return true;
      };
      while (ok && !final_seen) {
        const int slot = c & 1;
        if (!mbar_wait(B.tab_full + slot, (c >> 1) & 1, abort_flag, P.dev_status)) { ok = false; break; }
        const ChunkDesc d = desc[slot];
        mbar_arrive(B.tab_empty + slot);
        ++c;
        final_seen = (d.flags & kFlagFinal) != 0;
        const int ntiles = ceil_tiles(d.nkeys);
        for (int t = 0; t < ntiles; ++t, ++g) {
          const bool first = (d.flags & kFlagFirst) && t == 0;
          const bool last = (d.flags & kFlagLast) && t == ntiles - 1;
          if (first) {   // this unit's Q and dO have landed
            if (!mbar_wait(B.qd_full, u & 1, abort_flag, P.dev_status)) { ok = false; break; }
            ++u;
          }
          if (!mbar_wait(B.k_full + g % kStagesK, (g / kStagesK) & 1, abort_flag, P.dev_status) ||
              !mbar_wait(B.v_full + (g & 1), (g >> 1) & 1, abort_flag, P.dev_status)) {
            ok = false;
            break;
          }
          // S/dP buffer g&1 was last read by the softmax of tile g-2, whose
          // P/dS the dQ/dV/dK products of that tile (issued before this)
          // waited for
          tc_fence_after_sync();
          const uint32_t sb = (g & 1) * 128;
          const uint32_t k_addr = sbase + L::kKOff + (g % kStagesK) * L::kTileBytes;
          const uint32_t v_addr = sbase + L::kVOff + (g & 1) * L::kTileBytes;
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {   // K-dim: 16 columns of d per step
            const uint32_t off = (k >> 2) * L::kHalfBytes + (k & 3) * 32;
            const uint32_t toff = (k >> 2) * (kT * 128) + (k & 3) * 32;
            umma_ss(tmem + L::kSCol + sb, smem_desc_sw128(q_addr + off, 16, 1024), smem_desc_sw128(k_addr + toff, 16, 1024),
                    id_s, k > 0 ? 1u : 0u);
          }
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint32_t off = (k >> 2) * L::kHalfBytes + (k & 3) * 32;
            const uint32_t toff = (k >> 2) * (kT * 128) + (k & 3) * 32;
            umma_ss(tmem + L::kDPCol + sb, smem_desc_sw128(do_addr + off, 16, 1024),
                    smem_desc_sw128(v_addr + toff, 16, 1024), id_s, k > 0 ? 1u : 0u);
          }
          tc_commit(B.v_empty + (g & 1));
          tc_commit(B.s_full + (g & 1));
          // then the rest of the previous tile, once its P and dS are in
          // shared memory: the softmax of this tile overlaps those products
          if (pending && (!mbar_wait(B.p_ready, pg & 1, abort_flag, P.dev_status) || !issue_d(pg, p_first, p_last))) {
            ok = false;
            break;
          }
          pending = true;
          pg = g;
          p_first = first;
          p_last = last;
        }
        // The unit's last products go out now: the next unit needs this
        // unit's Q/dO buffers and its chunk may not be published before
        // the reducers have finished with this one.
        if (ok && pending && (d.flags & kFlagLast)) {
          if (!mbar_wait(B.p_ready, pg & 1, abort_flag, P.dev_status) || !issue_d(pg, p_first, p_last)) {
            ok = false;
            break;
          }
          pending = false;
        }
      }
      // every UMMA has completed before TMEM is released
      tc_commit(B.mma_done);
      mbar_wait(B.mma_done, 0, nullptr, P.dev_status);
    }
  } else if (warp < 4) {
    // ================================================= P and dS
    const int row = tid;   // head row == TMEM lane
    const int h = head0 + row;
    const bool row_ok = row < heads_here;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const float sink2 = (P.sink != nullptr && row_ok) ? P.sink[h] * kLog2e : -INFINITY;
    float dsink_acc = 0.f, lse2 = INFINITY, Dh = 0.f;
    int c = 0, g = 0, u = 0;
    bool ok = true, final_seen = false;
    while (ok && !final_seen) {
      const int slot = c & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(B.tab_full + slot, (c >> 1) & 1, abort_flag, P.dev_status))) break;
      const ChunkDesc d = desc[slot];
      mbar_arrive(B.tab_empty + slot);
      ++c;
      final_seen = (d.flags & kFlagFinal) != 0;
      const int ntiles = ceil_tiles(d.nkeys);
      for (int t = 0; t < ntiles; ++t, ++g) {
        if ((d.flags & kFlagFirst) && t == 0) {
          // unit prologue: D = dO . O (the saved BF16 O), the saved LSE,
          // and the sink's gradient term (once per query: by the slice that
          // holds the set's first key; empty slices do no work at all)
          if (!__all_sync(0xffffffffu, mbar_wait(B.qd_full, u & 1, abort_flag, P.dev_status))) {
            ok = false;
            break;
          }
          ++u;
          if (row_ok) {
            const int64_t qh = static_cast<int64_t>(d.i) * P.num_heads + h;
            const float lse = P.lse[qh];
            lse2 = lse * kLog2e;
            const uint4* orow = reinterpret_cast<const uint4*>(P.o + qh * D);
            uint4 ov[D / 8];
#pragma unroll
            for (int k = 0; k < D / 8; ++k) ov[k] = __ldg(orow + k);
            float acc = 0.f;
#pragma unroll
            for (int k = 0; k < D / 8; ++k) {
              const uint4 dv = *reinterpret_cast<const uint4*>(smem + L::kDOOff + (k >> 3) * L::kHalfBytes + row * 128 +
                                                               (((k & 7) ^ (row & 7)) << 4));
              acc += dot8_bf16(ov[k], dv);
            }
            Dh = acc;
            // an LSE of -inf (no keys, no sink) cannot reach here: the unit has keys
            if ((d.flags & kFlagSetStart) && sink2 > -INFINITY) dsink_acc -= exp2_approx(sink2 - lse2) * Dh;
          }
        }
        if (!__all_sync(0xffffffffu, mbar_wait(B.s_full + (g & 1), (g >> 1) & 1, abort_flag, P.dev_status))) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const int nv = min(kT, d.nkeys - t * kT);
        uint8_t* pbuf = smem + L::kPOff + row * 128;
        uint8_t* dsbuf = pbuf + L::kPBytes;
        bool stores_ok = true;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          uint32_t s[32], dp[32];
          tmem_ld32(lane_addr + L::kSCol + (g & 1) * 128 + 32 * hf, s);
          tmem_ld32(lane_addr + L::kDPCol + (g & 1) * 128 + 32 * hf, dp);
          tmem_ld_wait(s);
          tmem_ld_wait(dp);
          uint32_t pk[16], dk[16];
#pragma unroll
          for (int cc = 0; cc < 16; ++cc) {
            const int j = 32 * hf + 2 * cc;
            const float p0 = (j < nv && row_ok) ? exp2_approx(fmaf(__uint_as_float(s[2 * cc]), P.scale_log2, -lse2)) : 0.f;
            const float p1 =
                (j + 1 < nv && row_ok) ? exp2_approx(fmaf(__uint_as_float(s[2 * cc + 1]), P.scale_log2, -lse2)) : 0.f;
            const float d0 = p0 * (__uint_as_float(dp[2 * cc]) - Dh) * P.scale;
            const float d1 = p1 * (__uint_as_float(dp[2 * cc + 1]) - Dh) * P.scale;
            pk[cc] = pack_bf16x2(p0, p1);
            dk[cc] = pack_bf16x2(d0, d1);
          }
          // P/dS are free once the products of tile g-1 have completed:
          // the first half's exponentials do not wait for that
          if (hf == 0 &&
              !__all_sync(0xffffffffu, mbar_wait(B.pd_free, (g & 1) ^ 1, abort_flag, P.dev_status))) {
            stores_ok = false;
            break;
          }
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int chunk = 4 * hf + q;
            const int off = (chunk ^ (row & 7)) << 4;
            *reinterpret_cast<uint4*>(pbuf + off) = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
            *reinterpret_cast<uint4*>(dsbuf + off) = make_uint4(dk[4 * q], dk[4 * q + 1], dk[4 * q + 2], dk[4 * q + 3]);
          }
        }
        if (!stores_ok) {
          ok = false;
          break;
        }
        fence_proxy_async_smem();   // generic-proxy writes -> the UMMA's reads
        tc_fence_before_sync();
        mbar_arrive(B.p_ready);
      }
    }
    if (row_ok && P.dsink != nullptr && dsink_acc != 0.f) atomicAdd(P.dsink + h, dsink_acc);
  } else if (warp >= kRedWarp0) {
    // ================================================= gradient reductions
    // Thread r holds TMEM lane r: the d index r of dV^T/dK^T (keys along
    // the columns), the head row r of dQ. A dV or dK tile is written into
    // the staging tile as 64 key rows of d FP32 values; then each of the
    // first nv threads hands its key's row to the TMA unit as one bulk
    // reduction into the gradient pool. dQ leaves through the warp's 2 KB
    // stage as 16-byte vector reductions.
    const int r = tid - kRedWarp0 * 32;
    const int wq = warp - kRedWarp0;                   // this warp's 32 d / head rows
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    float* stg = reinterpret_cast<float*>(smem + L::kStageOff + wq * 2048);
    float* bulk = reinterpret_cast<float*>(smem + L::kBulkOff);
    const uint32_t bulk_addr = sbase + L::kBulkOff;
    uint32_t nsync = 0;
    // barrier of the 128 reducer threads (bounded: false once a wait gave up)
    auto rsync = [&]() -> bool {
      uint64_t* bar = B.red_sync + (nsync & 1);
      const uint32_t parity = (nsync >> 1) & 1;
      ++nsync;
      mbar_arrive(bar);
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, P.dev_status));
    };
    int c = 0, g = 0, ud = 0;
    bool ok = true, final_seen = false;
    while (ok && !final_seen) {
      const int slot = c & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(B.tab_full + slot, (c >> 1) & 1, abort_flag, P.dev_status))) break;
      const ChunkDesc d = desc[slot];
      final_seen = (d.flags & kFlagFinal) != 0;
      const uint32_t* t_rows = tab + slot * kChunkKeys;
      const int ntiles = ceil_tiles(d.nkeys);
      for (int t = 0; ok && t < ntiles; ++t, ++g) {
        if (!__all_sync(0xffffffffu, mbar_wait(B.g_full, g & 1, abort_flag, P.dev_status))) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const int nv = min(kT, d.nkeys - t * kT);
        // this thread's key row (threads r < nv hand one row each to the TMA)
        const uint32_t e = r < nv ? t_rows[t * kT + r] : kInvalidRow;
#pragma unroll 1
        for (int which = 0; which < 2; ++which) {   // dV, then dK
          // the staging tile is free once every reduction issued from it
          // has read it
          bulk_wait_read_all();
          if (!rsync()) {
            ok = false;
            break;
          }
#pragma unroll
          for (int hk = 0; hk < 2; ++hk) {
            uint32_t v[32];
            tmem_ld32(lane_addr + L::kGCol + which * kT + 32 * hk, v);
            tmem_ld_wait(v);
            if (r < D) {
#pragma unroll
              for (int kk = 0; kk < 32; ++kk) bulk[(32 * hk + kk) * D + r] = __uint_as_float(v[kk]);
            }
          }
          if (which == 1) {   // dV^T and dK^T have left TMEM
            tc_fence_before_sync();
            mbar_arrive(B.g_free);
          }
          fence_proxy_async_smem();   // generic-proxy writes -> the TMA's reads
          if (!rsync()) {
            ok = false;
            break;
          }
          if (e != kInvalidRow) {
            float* pool = which == 0 ? ((e & kRawBit) ? P.dv_raw : P.dv_cmp) : ((e & kRawBit) ? P.dk_raw : P.dk_cmp);
            bulk_reduce_add_f32(pool + static_cast<int64_t>(e & ~kRawBit) * D, bulk_addr + r * D * 4, D * 4);
          }
          bulk_commit_group();
        }
        if (!ok) break;
        if ((d.flags & kFlagLast) && t == ntiles - 1) {
          // dQ of the unit (head row r), added into dq: 16 columns of the
          // warp's 32 rows per pass through the stage, then 8 rows x 64
          // contiguous bytes per vector reduction
          if (!__all_sync(0xffffffffu, mbar_wait(B.dq_full, ud & 1, abort_flag, P.dev_status))) {
            ok = false;
            break;
          }
          ++ud;
          tc_fence_after_sync();
          float* dq_base = P.dq + (static_cast<int64_t>(d.i) * P.num_heads + head0 + wq * 32) * D;
          const int swz = (lane >> 1) & 3;
#pragma unroll 1
          for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t v[32];
            tmem_ld32(lane_addr + L::kDQCol + c0, v);
            tmem_ld_wait(v);
            if (c0 + 32 == D) {
              tc_fence_before_sync();
              mbar_arrive(B.dq_free);
            }
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
              float4* row = reinterpret_cast<float4*>(stg + lane * 16);
#pragma unroll
              for (int q = 0; q < 4; ++q)
                row[q ^ swz] = make_float4(__uint_as_float(v[16 * hf + 4 * q]), __uint_as_float(v[16 * hf + 4 * q + 1]),
                                           __uint_as_float(v[16 * hf + 4 * q + 2]), __uint_as_float(v[16 * hf + 4 * q + 3]));
              __syncwarp();
              float4 x[4];
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const int rr = 8 * k + (lane >> 2), piece = lane & 3;
                x[k] = reinterpret_cast<const float4*>(stg + rr * 16)[piece ^ ((rr >> 1) & 3)];
              }
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const int rr = 8 * k + (lane >> 2), piece = lane & 3;
                if (wq * 32 + rr < heads_here)
                  red_add_v4_f32(dq_base + static_cast<int64_t>(rr) * D + c0 + 16 * hf + 4 * piece, x[k]);
              }
              __syncwarp();
            }
          }
        }
      }
      mbar_arrive(B.tab_empty + slot);
      ++c;
    }
    bulk_wait_all();   // every bulk reduction has completed
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
    cudaError_t err =
        cudaFuncSetAttribute(sparse_sink_attn_bwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes);
    if (err != cudaSuccess) return err;
    configured = true;
  }
  const int64_t units = static_cast<int64_t>(P.n_queries) * P.num_splits;
  const int64_t slots = std::max<int64_t>(1, static_cast<int64_t>(device_sm_count()) / head_tiles);
  dim3 grid(static_cast<unsigned>(std::min<int64_t>(units, slots)), head_tiles);
  sparse_sink_attn_bwd_kernel<D><<<grid, kThreads, L::kBytes, stream>>>(P);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_sparse_sink_attn_bwd(const AttnArgs& a, cudaStream_t stream) {
  if (a.n_queries == 0) return cudaSuccess;
  Params P;
  memset(&P, 0, sizeof P);
  if (tensor_map_encoder() == nullptr) return cudaErrorNotSupported;
  P.q_box_rows = std::min(128, a.num_heads);
  const int64_t raw_rows = a.raw_num_pages * a.raw_page_size;
  if (!encode_q(&P.tm_q, a.q, a.n_queries, a.num_heads, a.head_dim, a.q_stride_tok, a.q_stride_head,
                P.q_box_rows) ||
      !encode_q(&P.tm_do, a.dout, a.n_queries, a.num_heads, a.head_dim,
                static_cast<int64_t>(a.num_heads) * a.head_dim, a.head_dim, P.q_box_rows) ||
      !encode_pool(&P.tm_k_raw, a.k_raw, raw_rows, a.head_dim) ||
      !encode_pool(&P.tm_v_raw, a.v_raw, raw_rows, a.head_dim))
    return cudaErrorInvalidValue;
  if (a.pt_cmp != nullptr) {
    const int64_t cmp_rows = a.cmp_num_pages * a.cmp_page_size;
    if (!encode_pool(&P.tm_k_cmp, a.k_cmp, cmp_rows, a.head_dim) ||
        !encode_pool(&P.tm_v_cmp, a.v_cmp, cmp_rows, a.head_dim))
      return cudaErrorInvalidValue;
  }
  P.n_queries = a.n_queries;
  P.num_heads = a.num_heads;
  P.raw_pages = a.raw_num_pages;
  P.raw_ps_log2 = log2_exact(a.raw_page_size);
  P.pt_raw = a.pt_raw;
  P.pt_raw_cols = a.pt_raw_cols;
  P.cmp_pages = a.pt_cmp ? a.cmp_num_pages : 0;
  P.cmp_ps_log2 = a.pt_cmp ? log2_exact(a.cmp_page_size) : 0;
  P.pt_cmp = a.pt_cmp;
  P.pt_cmp_cols = a.pt_cmp ? a.pt_cmp_cols : 0;
  P.req = a.req;
  P.n_requests = a.n_requests;
  P.indptr = a.indptr;
  P.indices = a.indices;
  P.set_pos = a.set_pos;
  P.set_window = a.set_window;
  P.set_ratio = a.set_ratio;
  P.set_topk = a.set_topk;
  P.set_topk_width = a.set_topk_width;
  P.sink = a.sink;
  P.scale = a.scale;
  P.scale_log2 = static_cast<float>(static_cast<double>(a.scale) * 1.4426950408889634);
  P.o = a.o_saved;
  P.lse = a.lse_saved;
  P.dq = a.dq;
  P.dk_raw = a.dk_raw;
  P.dv_raw = a.dv_raw;
  P.dk_cmp = a.dk_cmp;
  P.dv_cmp = a.dv_cmp;
  P.dsink = a.dsink;
  P.num_splits = a.num_splits;
  P.dev_status = a.dev_status;
  P.wait_ns = kWaitTimeoutNs;
  const int head_tiles = (a.num_heads + 127) / 128;
  if (a.head_dim == 128) return launch_d<128>(P, head_tiles, stream);
  return launch_d<64>(P, head_tiles, stream);
}

}  // namespace spa
