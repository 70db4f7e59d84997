// Sparse paged attention with an attention sink at the DSV4-Flash attention
// shape: head width d = 512, 32 query heads per tile sharing every K/V row.
//
// Page "Roadmap item 24 - joint compressed/window attention with sink",
// section "Reuse and arithmetic": the fixed H32 launch recipe; compressed
// KV, the full recent window and the sink share one softmax denominator;
// the sink has no V; P and O are BF16 and LSE is the FP32 natural log of
// the denominator. The review notes on the packed joint KV gather of the
// same page give the 512-wide head (584 bytes per packed token, decoded to
// BF16 rows by spa_unpack_d512_pages before this call).
//
// With 32 heads and d = 512 the products are transposed so that the tensor
// cores keep M = 128 and the accumulators stay small:
//   S^T[key, h] = sum_e K[key, e] Q[h, e]     M = 128 keys, N = 32 heads, K = 512
//   O^T[e, h]  += sum_key V[key, e] P[h, key]  M = 128 columns of d (4 blocks), N = 32, K = 128 keys
// TMEM holds two S^T buffers (32 columns each) and the four O^T blocks
// (128 columns). K and V rows stream through shared memory in chunks of 64
// columns of d (one 128-byte swizzle atom per row): a K chunk [128 keys x
// 64] is the K-major A operand of four S^T products; two V chunks [128
// keys x 128] are the M-major A operand of eight O^T products. Q [32 x 512]
// stays in shared memory as the K-major B operand of S^T; P^T [32 heads x
// 128 keys] is written by the softmax threads as the K-major B operand of
// O^T. At 32 heads a key row carries 32 x 4 x 512 FLOPs for 2 KB of K and V:
// 32 FLOP/B, so this shape is bound by moving rows, not by the tensor cores.
//
// Softmax thread t owns TMEM lane t: key t of the tile in S^T, column t of d
// (per 128-column block) in O^T. The running max m[h] is the same in every
// thread; each thread keeps its own partial row sums l[h], added up at the
// end of the unit. As in the 128-head kernel, P is taken with the running
// max as it stands and a tile is redone with its exact per-head max only
// when some P leaves a fixed bound (then O^T columns are rescaled).
//
// Warp roles (512 threads, one CTA per SM):
//   warps 0-3   softmax + epilogue
//   warp  4     TMEM allocation; lane 0 issues every UMMA and commit
//   warp  5     resolver (keys -> physical rows, as in the 128-head kernel)
//   warp  6     Q: eight TMA boxes per unit
//   warps 8-11  K chunks, warps 12-15 V chunk pairs: 16-byte cp.async
// Split-KV: the slices of a query are the CTAs of one cluster (up to 8) and
// merge exactly through distributed shared memory.
#include <cmath>
#include <cstring>

#include "attn_common.cuh"

namespace spa {
namespace {

using namespace attn;

constexpr int kD = 512;
constexpr int kHT = 32;                    // heads per tile (N of both products)
constexpr int kTk = 128;                   // keys per tile (M of S^T)
constexpr int kNChunks = kD / 64;          // 64-column chunks of a row
constexpr int kChunkBytes = kTk * 128;     // [128 rows][64 columns] BF16
constexpr int kKStages = 4;                // K ring: single chunks
constexpr int kVStages = 2;                // V ring: chunk pairs (a 128-column block of d)
constexpr int kOBlocks = kD / 128;
constexpr int kThreads = 512;
constexpr int kSoftThreads = 128;
constexpr int kMmaWarp = 4;
constexpr int kResolverWarp = 5;
constexpr int kQWarp = 6;
constexpr int kKGroupWarp0 = 8;
constexpr int kVGroupWarp0 = 12;
constexpr int kGroupThreads = 128;
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kSCol = 0;              // S^T buffers: [2][32]
constexpr uint32_t kOCol = 64;             // O^T blocks: [4][32]
constexpr float kSpecBound = 65536.0f;
// registers per thread after the split (one 512-thread CTA per SM: 4 x 128)
constexpr uint32_t kRegSoftmax = 232;
constexpr uint32_t kRegControl = 120;
constexpr uint32_t kRegGather = 80;
static_assert(kRegSoftmax + kRegControl + 2 * kRegGather <= 4 * 128, "register split exceeds the launch");
// consumers of a chunk descriptor: K and V groups, MMA thread, softmax, Q warp
constexpr uint32_t kTabConsumers = 2 * kGroupThreads + 1 + kSoftThreads + 32;

struct Params {
  CUtensorMap tm_q;   // 3D {512, H, N}, box {64, q_box_rows, 1}
  const uint8_t* k_raw;
  const uint8_t* v_raw;
  const uint8_t* k_cmp;
  const uint8_t* v_cmp;
  int32_t q_box_rows;   // min(32, num_heads)
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
  float scale_log2;
  uint16_t* out;
  float* lse;
  int32_t num_splits;   // slices per query; > 1: one cluster of that many CTAs per query
  uint32_t* dev_status;
  uint64_t wait_ns;
  int32_t stall;        // testing: every CTA waits on a barrier nothing arrives at
};

struct Layout {
  static constexpr int kQOff = 0;                                   // [8][32 rows][128 B]
  static constexpr int kKOff = kQOff + kNChunks * kHT * 128;        // [4][16 KB]
  static constexpr int kVOff = kKOff + kKStages * kChunkBytes;      // [2][32 KB]
  static constexpr int kPOff = kVOff + kVStages * 2 * kChunkBytes;  // [2][2 halves][32 rows][128 B]
  static constexpr int kPBytes = 2 * kHT * 128;
  static constexpr int kTabOff = kPOff + 2 * kPBytes;               // [2][kChunkKeys] u32
  static constexpr int kDescOff = kTabOff + 2 * kChunkKeys * 4;
  static constexpr int kRedOff = kDescOff + 2 * static_cast<int>(sizeof(ChunkDesc));   // [32][128] f32
  static constexpr int kStageOff = kRedOff + kHT * kSoftThreads * 4;                  // [4 warps][2 KB]
  static constexpr int kHeadOff = kStageOff + 4 * 2048;             // [32] f32 each: sink, m, 1/l or weight
  static constexpr int kMlOff = kHeadOff + 3 * kHT * 4;             // [32] float2: (m, l) for the merge
  static constexpr int kMaxOff = kMlOff + kHT * 8;                  // [4 warps][32] f32: tile maxima
  static constexpr int kBarOff = kMaxOff + 4 * kHT * 4;
  static constexpr int kNumBars = 2 + 2 + 2 + 2 * kKStages + 2 * kVStages + 2 + 2 + 2 + 2 + 1 + 1 + 1 + 2;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 48 + 1024;   // misc: TMEM slot, abort, have_o, votes, stall barrier at +32
  static_assert(kBytes <= 227 * 1024, "shared memory");
  static_assert(kKStages * kChunkBytes == kHT * kD * 4, "the merge reuses the K ring for [32][512] FP32");
};

struct Bars {
  uint64_t *tab_full, *tab_empty;   // [2]
  uint64_t *q_full, *q_empty;
  uint64_t *k_full, *k_empty;       // [kKStages]
  uint64_t *v_full, *v_empty;       // [kVStages]
  uint64_t *s_full, *s_free;        // [2]
  uint64_t *p_ready, *p_free;       // [2]
  uint64_t *o_done, *o_free, *mma_done;
  uint64_t* soft_sync;              // [2]
};

// Bounded barrier of the 128 softmax threads; the two mbarriers alternate.
struct SoftSync {
  uint64_t* bars;
  volatile int* abort_flag;
  uint32_t* dev_status;
  uint64_t wait_ns;
  uint32_t n = 0;
  __device__ bool operator()() {
    uint64_t* bar = bars + (n & 1);
    const uint32_t parity = (n >> 1) & 1;
    ++n;
    mbar_arrive(bar);
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, dev_status, wait_ns));
  }
};

// Bytes of the merge's receive slots [S][32 heads][widest column range]
// FP16, the largest over 2..8 slices.
constexpr int merge_rx_bytes_max() {
  int m = 0;
  for (int S = 2; S <= kAttnMaxClusterSplits; ++S) {
    const int per = (kD / S) & ~7;
    const int b = S * kHT * (kD - (S - 1) * per) * 2;
    m = b > m ? b : m;
  }
  return m;
}

// End of every role (inlined into each): the cluster merge of the slices
// by the softmax threads, the cluster barriers for every warp, TMEM freed
// by the MMA warp last.
__device__ __forceinline__ void cta_finish(const Params& P, bool soft, uint8_t* smem, uint32_t sbase, uint32_t tmem,
                                           int tid, int warp, int head0, int heads_here, SoftSync* ss) {
  using L = Layout;
  __syncwarp();
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const int S = P.num_splits;
  if (S > 1) {
    // Exact merge of the S slices of query i (page "[WS2] Add CP-aware
    // Attention contract and dispatch metadata", Summary: the deterministic
    // (out, lse) merge): w_s = 2^(m_s - M) / L per head. CTA r owns columns
    // [r*per, ...) of d. Each CTA scales its O^T by its weights into its own
    // shared memory as [head][d] FP32, then stores every 8-column piece as
    // FP16 (16 bytes) straight into its owner's receive slots (posted
    // remote stores, slot = the sender's rank; its own columns with local
    // stores); after the second cluster barrier each owner sums its slots
    // in FP32 and writes BF16 O. FP16 keeps more bits than the BF16 output
    // and halves the remote bytes. Nothing is read or written remotely
    // after that barrier, so no third one is needed.
    const int rank = static_cast<int>(cluster_ctarank());
    const int i = static_cast<int>(blockIdx.x / S);
    const int per = (kD / S) & ~7;   // 8-column pieces; the last rank takes the rest
    const int own_e0 = rank * per, own_e1 = rank == S - 1 ? kD : own_e0 + per;
    const int span = kD - (S - 1) * per;   // the widest range (the last rank's)
    float* head_w = reinterpret_cast<float*>(smem + L::kHeadOff + 2 * kHT * 4);
    const bool have_o = *reinterpret_cast<const int*>(smem + L::kMiscOff + 8) != 0;
    // receive slots [S][32 heads][span] FP16 after the K ring (idle by now)
    static_assert(L::kPOff + 2 * L::kPBytes - L::kVOff >= merge_rx_bytes_max(), "receive slots fit the idle V ring and P");
    const uint32_t rx_addr = sbase + L::kVOff;
    __syncwarp();
    cluster_sync_all();   // every slice's (m, l) is in place
    if (soft) {
      if (tid < kHT) {
        const int h = tid;
        float2 ml[kAttnMaxClusterSplits];
#pragma unroll
        for (int s = 0; s < kAttnMaxClusterSplits; ++s)
          ml[s] = s < S ? ld_dsmem_f2(dsmem_addr(sbase + L::kMlOff + h * 8, s)) : make_float2(-INFINITY, 0.f);
        float M = -INFINITY;
#pragma unroll
        for (int s = 0; s < kAttnMaxClusterSplits; ++s)
          if (ml[s].y > 0.f) M = fmaxf(M, ml[s].x);
        float Lsum = 0.f, w_own = 0.f;
#pragma unroll
        for (int s = 0; s < kAttnMaxClusterSplits; ++s) {
          const float w = (ml[s].y > 0.f) ? exp2_approx(ml[s].x - M) : 0.f;
          Lsum += w * ml[s].y;
          if (s == rank) w_own = w;
        }
        head_w[h] = Lsum > 0.f ? w_own / Lsum : 0.f;
        if (rank == 0 && h < heads_here)
          P.lse[static_cast<int64_t>(i) * P.num_heads + head0 + h] =
              Lsum > 0.f ? (M + log2_approx(Lsum)) * kLn2 : -INFINITY;
      }
      (*ss)();
      float w[kHT];
#pragma unroll
      for (int h = 0; h < kHT; ++h) w[h] = head_w[h];
      float* wo = reinterpret_cast<float*>(smem + L::kKOff);   // [32][512] FP32
      const uint32_t lane_addr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
#pragma unroll 1
      for (int b = 0; b < kOBlocks; ++b) {
        uint32_t o[32];
        if (have_o) {
          tmem_ld32(lane_addr + kOCol + 32 * b, o);
          tmem_ld_wait(o);
        } else {
#pragma unroll
          for (int h = 0; h < kHT; ++h) o[h] = 0u;
        }
#pragma unroll
        for (int h = 0; h < kHT; ++h) wo[h * kD + 128 * b + tid] = __uint_as_float(o[h]) * w[h];
      }
      (*ss)();   // this CTA's scaled rows are in place
      for (int item = tid; item < kHT * (kD / 8); item += kSoftThreads) {
        const int h = item / (kD / 8), e = 8 * (item % (kD / 8));
        const int owner = min(e / per, S - 1);
        const int e_rel = e - owner * per;
        const float4 a = *reinterpret_cast<const float4*>(wo + h * kD + e);
        const float4 b = *reinterpret_cast<const float4*>(wo + h * kD + e + 4);
        const uint4 v = make_uint4(pack_f16x2(a.x, a.y), pack_f16x2(a.z, a.w), pack_f16x2(b.x, b.y), pack_f16x2(b.z, b.w));
        const uint32_t slot = rx_addr + static_cast<uint32_t>(((rank * kHT + h) * span + e_rel) * 2);
        if (owner == rank)
          *reinterpret_cast<uint4*>(smem + (slot - sbase)) = v;
        else
          st_dsmem_f4(dsmem_addr(slot, owner), make_float4(__uint_as_float(v.x), __uint_as_float(v.y),
                                                           __uint_as_float(v.z), __uint_as_float(v.w)));
      }
    }
    __syncwarp();
    cluster_sync_all();   // every slice's pieces have arrived
    if (soft) {
      const int n8 = (own_e1 - own_e0) / 8;
      const uint8_t* rx = smem + L::kVOff;
      for (int item = tid; item < kHT * n8; item += kSoftThreads) {
        const int h = item / n8, e_rel = 8 * (item % n8);
        if (h >= heads_here) continue;
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int s = 0; s < S; ++s) {
          const uint4 v = *reinterpret_cast<const uint4*>(rx + ((s * kHT + h) * span + e_rel) * 2);
          const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float2 f = unpack_f16x2(w4[k]);
            acc[2 * k] += f.x;
            acc[2 * k + 1] += f.y;
          }
        }
        *reinterpret_cast<uint4*>(P.out + (static_cast<int64_t>(i) * P.num_heads + head0 + h) * kD + own_e0 + e_rel) =
            make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]), pack_bf16x2(acc[4], acc[5]),
                       pack_bf16x2(acc[6], acc[7]));
      }
    }
  }
  if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

__global__ void __launch_bounds__(kThreads, 1) sparse_sink_attn_d512_kernel(const __grid_constant__ Params P) {
  using L = Layout;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bar0 = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  Bars B;
  B.tab_full = bar0;
  B.tab_empty = bar0 + 2;
  B.q_full = bar0 + 4;
  B.q_empty = bar0 + 5;
  B.k_full = bar0 + 6;
  B.k_empty = B.k_full + kKStages;
  B.v_full = B.k_empty + kKStages;
  B.v_empty = B.v_full + kVStages;
  B.s_full = B.v_empty + kVStages;
  B.s_free = B.s_full + 2;
  B.p_ready = B.s_free + 2;
  B.p_free = B.p_ready + 2;
  B.o_done = B.p_free + 2;
  B.o_free = B.o_done + 1;
  B.mma_done = B.o_free + 1;
  B.soft_sync = B.mma_done + 1;
  uint32_t* tab = reinterpret_cast<uint32_t*>(smem + L::kTabOff);
  ChunkDesc* desc = reinterpret_cast<ChunkDesc*>(smem + L::kDescOff);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int S = P.num_splits;
  const int head0 = blockIdx.y * kHT;
  const int heads_here = min(kHT, P.num_heads - head0);
  float* head_sink = reinterpret_cast<float*>(smem + L::kHeadOff);
  float* head_m = head_sink + kHT;
  float* head_x = head_m + kHT;   // 1/l (epilogue) or merge weight

  // ---- setup
  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(B.tab_full + s, 32);
      mbar_init(B.tab_empty + s, kTabConsumers);
      mbar_init(B.s_full + s, 1);
      mbar_init(B.s_free + s, kSoftThreads);
      mbar_init(B.p_ready + s, kSoftThreads);
      mbar_init(B.p_free + s, 1);
      mbar_init(B.soft_sync + s, kSoftThreads);
    }
    mbar_init(B.q_full, 1);
    mbar_init(B.q_empty, 1);
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(B.k_full + s, kGroupThreads);
      mbar_init(B.k_empty + s, 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(B.v_full + s, kGroupThreads);
      mbar_init(B.v_empty + s, 1);
    }
    mbar_init(B.o_done, 1);
    mbar_init(B.o_free, kSoftThreads);
    mbar_init(B.mma_done, 1);
    *abort_flag = 0;
    *reinterpret_cast<int*>(smem + L::kMiscOff + 8) = 0;
    for (int k = 0; k < 3; ++k) reinterpret_cast<uint32_t*>(smem + L::kMiscOff + 16)[k] = 0u;
    mbar_init(reinterpret_cast<uint64_t*>(smem + L::kMiscOff + 32), 1);   // never arrived at
    mbar_init_fence();
  }
  if (tid < kHT) {
    const int h = head0 + tid;
    head_sink[tid] = (P.sink != nullptr && tid < heads_here) ? P.sink[h] * kLog2e : -INFINITY;
  }
  // Q rows past the heads of this tile are never written by the TMA: zero
  // them once so that those S^T columns stay finite (they are masked)
  if (P.q_box_rows < kHT) {
    for (int idx = tid; idx < kNChunks * (kHT - P.q_box_rows) * 8; idx += kThreads) {
      const int blk = idx / ((kHT - P.q_box_rows) * 8), rest = idx % ((kHT - P.q_box_rows) * 8);
      const int row = P.q_box_rows + rest / 8, ch = rest % 8;
      *reinterpret_cast<uint4*>(smem + L::kQOff + blk * (kHT * 128) + row * 128 + ch * 16) =
          make_uint4(0u, 0u, 0u, 0u);
    }
    fence_proxy_async_smem();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  // everything above is private to the CTA; every global read below may
  // depend on the previous kernel of the stream (the sets, the pools, Q)
  grid_dep_wait();
  SoftSync ss{B.soft_sync, abort_flag, P.dev_status, P.wait_ns};

  // one setmaxnreg per warpgroup, dominating all of its roles
  if (warp >= 4 && warp < 8) {
    warpgroup_reg_dealloc<kRegControl>();
    if (warp == kResolverWarp) {
      // ================================================= resolver
      // testing stall: a wait that only its limit ends, then the CTA unwinds
      if (P.stall) mbar_wait(reinterpret_cast<uint64_t*>(smem + L::kMiscOff + 32), 0, abort_flag, P.dev_status, P.wait_ns);
      resolver_loop(P, S, tab, desc, B.tab_full, B.tab_empty, abort_flag, lane);
      cta_finish(P, false, smem, sbase, tmem, tid, warp, head0, heads_here, &ss);
    } else if (warp == kQWarp) {
      // ================================================= Q loader
      // The CTA's first unit is unit blockIdx.x (units are strided over the
      // CTAs): its Q is loaded at once, while the resolver fetches its keys.
      int c = 0, qc = 1;
      bool final_seen = false, first_issued = true;
      if (lane == 0) {
        mbar_arrive_expect_tx(B.q_full, P.q_box_rows * 128 * kNChunks);
        for (int cb = 0; cb < kNChunks; ++cb)
          tma_load_3d(sbase + L::kQOff + cb * (kHT * 128), &P.tm_q, B.q_full, cb * 64, head0,
                      static_cast<int32_t>(blockIdx.x / S));
      }
      while (!final_seen) {
        const int slot = c & 1;
        if (!mbar_wait(B.tab_full + slot, (c >> 1) & 1, abort_flag, P.dev_status, P.wait_ns)) break;
        const ChunkDesc d = desc[slot];
        final_seen = (d.flags & kFlagFinal) != 0;
        bool ok = true;
        if ((d.flags & kFlagFirst) && first_issued) {
          first_issued = false;   // the first unit's Q is on its way
        } else if (d.flags & kFlagFirst) {
          // the previous unit's last S^T product has read Q
          ok = mbar_wait(B.q_empty, (qc & 1) ^ 1, abort_flag, P.dev_status, P.wait_ns);
          if (ok && lane == 0) {
            mbar_arrive_expect_tx(B.q_full, P.q_box_rows * 128 * kNChunks);
            for (int cb = 0; cb < kNChunks; ++cb)
              tma_load_3d(sbase + L::kQOff + cb * (kHT * 128), &P.tm_q, B.q_full, cb * 64, head0, d.i);
          }
          if (ok) ++qc;
        }
        __syncwarp();
        mbar_arrive(B.tab_empty + slot);
        ++c;
        if (!ok) break;
      }
      if (qc > 0) mbar_wait(B.q_full, (qc - 1) & 1, nullptr, P.dev_status);
      cta_finish(P, false, smem, sbase, tmem, tid, warp, head0, heads_here, &ss);
    } else if (warp == kMmaWarp) {
      // ================================================= UMMA issuer
      // S^T of tile g is issued before O^T of tile g-1, so the softmax of
      // tile g overlaps the O^T products of tile g-1.
      if (lane == 0) {
        constexpr uint32_t idesc_s = idesc_bf16_f32_ab(kTk, kHT, 0, 0);
        constexpr uint32_t idesc_o = idesc_bf16_f32_ab(128, kHT, 1, 0);
        int c = 0, g = 0, nk = 0, nvp = 0, u = 0, uo = 0;
        bool ok = true, final_seen = false;
        int pend_g = -1;
        bool pend_first = false, pend_last = false;
        auto issue_o = [&]() -> bool {   // O^T += V^T P^T of tile pend_g
          if (!mbar_wait(B.p_ready + (pend_g & 1), (pend_g >> 1) & 1, abort_flag, P.dev_status, P.wait_ns))
            return false;
          if (pend_first) {   // the previous unit's epilogue has read O^T
            if (!mbar_wait(B.o_free, (uo & 1) ^ 1, abort_flag, P.dev_status, P.wait_ns)) return false;
            ++uo;
          }
          tc_fence_after_sync();
          const uint32_t p_addr = sbase + L::kPOff + (pend_g & 1) * L::kPBytes;
          for (int b = 0; b < kOBlocks; ++b, ++nvp) {
            const int st = nvp % kVStages;
            if (!mbar_wait(B.v_full + st, (nvp / kVStages) & 1, abort_flag, P.dev_status, P.wait_ns)) return false;
            fence_proxy_async_smem();
            tc_fence_after_sync();
            const uint32_t v_addr = sbase + L::kVOff + st * (2 * kChunkBytes);
  #pragma unroll
            for (int kk = 0; kk < kTk / 16; ++kk) {
              const uint64_t a = smem_desc_sw128(v_addr + kk * 16 * 128, kChunkBytes, 1024);
              const uint64_t bd = smem_desc_sw128(p_addr + (kk >> 2) * (kHT * 128) + (kk & 3) * 32, 16, 1024);
              umma_ss(tmem + kOCol + 32 * b, a, bd, idesc_o, (!pend_first || kk > 0) ? 1u : 0u);
            }
            tc_commit(B.v_empty + st);
          }
          tc_commit(B.p_free + (pend_g & 1));
          if (pend_last) tc_commit(B.o_done);
          pend_g = -1;
          return true;
        };
        while (ok && !final_seen) {
          const int slot = c & 1;
          if (!mbar_wait(B.tab_full + slot, (c >> 1) & 1, abort_flag, P.dev_status, P.wait_ns)) { ok = false; break; }
          const ChunkDesc d = desc[slot];
          mbar_arrive(B.tab_empty + slot);
          ++c;
          final_seen = (d.flags & kFlagFinal) != 0;
          const int ntiles = (d.nkeys + kTk - 1) / kTk;
          if (d.flags & kFlagFirst) {
            // finish the previous unit before waiting for this unit's Q
            if (pend_g >= 0 && !issue_o()) { ok = false; break; }
            if (!mbar_wait(B.q_full, u & 1, abort_flag, P.dev_status, P.wait_ns)) { ok = false; break; }
            ++u;
          }
          for (int t = 0; t < ntiles; ++t, ++g) {
            const int sb = g & 1;
            if (!mbar_wait(B.s_free + sb, ((g >> 1) & 1) ^ 1, abort_flag, P.dev_status, P.wait_ns)) { ok = false; break; }
            tc_fence_after_sync();
            for (int cc = 0; cc < kNChunks; ++cc, ++nk) {
              const int st = nk % kKStages;
              if (!mbar_wait(B.k_full + st, (nk / kKStages) & 1, abort_flag, P.dev_status, P.wait_ns)) { ok = false; break; }
              fence_proxy_async_smem();   // the copies' rows, landed in the generic proxy -> the UMMA reads
              tc_fence_after_sync();
              const uint32_t k_addr = sbase + L::kKOff + st * kChunkBytes;
              const uint32_t q_addr = sbase + L::kQOff + cc * (kHT * 128);
  #pragma unroll
              for (int k = 0; k < 4; ++k)
                umma_ss(tmem + kSCol + 32 * sb, smem_desc_sw128(k_addr + k * 32, 16, 1024),
                        smem_desc_sw128(q_addr + k * 32, 16, 1024), idesc_s, (cc > 0 || k > 0) ? 1u : 0u);
              tc_commit(B.k_empty + st);
            }
            if (!ok) break;
            tc_commit(B.s_full + sb);
            const bool first = (d.flags & kFlagFirst) && t == 0;
            const bool last = (d.flags & kFlagLast) && t == ntiles - 1;
            if (last) tc_commit(B.q_empty);
            if (pend_g >= 0 && !issue_o()) { ok = false; break; }
            pend_g = g;
            pend_first = first;
            pend_last = last;
          }
          // an empty unit has no S^T product to release its Q
          if (ok && ntiles == 0 && (d.flags & kFlagLast)) tc_commit(B.q_empty);
        }
        if (ok && pend_g >= 0) issue_o();
        tc_commit(B.mma_done);
        mbar_wait(B.mma_done, 0, nullptr, P.dev_status);
      }
      cta_finish(P, false, smem, sbase, tmem, tid, warp, head0, heads_here, &ss);
    } else {
      cta_finish(P, false, smem, sbase, tmem, tid, warp, head0, heads_here, &ss);
    }
  } else if (warp >= kKGroupWarp0) {
    warpgroup_reg_dealloc<kRegGather>();
    // ================================================= K chunks / V chunk pairs (cp.async)
    // K: a chunk is columns [64c, 64c+64) of the tile's 128 rows; lane l
    // copies 16-byte piece l%8 of rows l/8 + 4j of its warp's 32 rows.
    // V: a pair is columns [128b, 128b+128); lane l copies piece l%16 of
    // rows l/16 + 2j. Piece p of row r lands at (p/8)*16 KB + r*128 +
    // ((p%8) ^ (r%8))*16: the 128-byte swizzle that both the K-major S^T
    // operand and the M-major O^T operand read. Each thread's copies of a
    // stage complete into the stage's barrier by themselves
    // (cp.async.mbarrier.arrive.noinc: one arrival per thread once its
    // copies have landed), so a thread never waits for its own copies and
    // every free stage is in flight; the UMMA issuer orders the landed rows
    // before its tensor-core reads with fence.proxy.async after the wait.
    // (Handing a stage over only after the next one was issued, waiting for
    // the copies, kept one stage in flight: about 1 us per 16 KB chunk.)
    const bool is_k = warp < kVGroupWarp0;
    const int gw = warp - (is_k ? kKGroupWarp0 : kVGroupWarp0);
    const int nst = is_k ? kKStages : kVStages;
    const int per_tile = is_k ? kNChunks : kOBlocks;
    const int stage_bytes = is_k ? kChunkBytes : 2 * kChunkBytes;
    uint64_t* full = is_k ? B.k_full : B.v_full;
    uint64_t* empty = is_k ? B.k_empty : B.v_empty;
    const uint8_t* pool_raw = is_k ? P.k_raw : P.v_raw;
    const uint8_t* pool_cmp = is_k ? P.k_cmp : P.v_cmp;
    const uint32_t ring = sbase + (is_k ? L::kKOff : L::kVOff);
    const int pieces = is_k ? 8 : 16;           // 16-byte pieces per row per stage
    const int rows_per_instr = 32 / pieces;
    const int piece = lane % pieces, rsub = lane / pieces;
    const uint32_t col_off = static_cast<uint32_t>((piece / 8) * kChunkBytes);
    const int p8 = piece % 8;
int c = 0, n = 0;
    bool final_seen = false;
    while (!final_seen) {
      const int slot = c & 1;
if (!mbar_wait(B.tab_full + slot, (c >> 1) & 1, abort_flag, P.dev_status, P.wait_ns)) break;
      const ChunkDesc d = desc[slot];
      final_seen = (d.flags & kFlagFinal) != 0;
      const uint32_t* t_rows = tab + slot * kChunkKeys;
      const int ntiles = (d.nkeys + kTk - 1) / kTk;
      bool ok = true;
      for (int t = 0; ok && t < ntiles; ++t) {
        const int nv = min(kTk, d.nkeys - t * kTk);
        const uint32_t* trow = t_rows + t * kTk;
        for (int part = 0; part < per_tile; ++part, ++n) {
          const int stage = n % nst;
          const uint32_t par = ((n / nst) & 1) ^ 1;
if (!mbar_wait(empty + stage, par, abort_flag, P.dev_status, P.wait_ns)) { ok = false; break; }
          const uint32_t stage_base = ring + stage * stage_bytes + col_off;
          const int64_t col_bytes = static_cast<int64_t>(part) * (is_k ? 128 : 256) + piece * 16;
#pragma unroll 4
          for (int j = 0; j < 32 / rows_per_instr; ++j) {
            const int r = gw * 32 + j * rows_per_instr + rsub;
            const uint32_t e = r < nv ? trow[r] : kInvalidRow;
            const uint8_t* base = (e & kRawBit) ? pool_raw : pool_cmp;
            const bool valid = e != kInvalidRow && base != nullptr;
            const uint8_t* src = valid ? base + static_cast<int64_t>(e & ~kRawBit) * (kD * 2) + col_bytes : pool_raw;
            cp_async16(stage_base + r * 128 + ((p8 ^ (r & 7)) << 4), src, valid ? 16u : 0u);
          }
          cp_async_arrive_noinc(full + stage);
        }
      }
      mbar_arrive(B.tab_empty + slot);
      ++c;
      if (!ok) break;
    }
    cp_async_wait_all();   // no copy of this thread is in flight when the CTA leaves
    cta_finish(P, false, smem, sbase, tmem, tid, warp, head0, heads_here, &ss);
  } else {
    warpgroup_reg_alloc<kRegSoftmax>();
    // ================================================= softmax + epilogue
    const int row = tid;   // key of S^T / column of d within an O^T block
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    float* red = reinterpret_cast<float*>(smem + L::kRedOff);      // [32][128]
    float* tmax_w = reinterpret_cast<float*>(smem + L::kMaxOff);   // [4][32]
    uint8_t* pbuf0 = smem + L::kPOff;
    uint8_t* stage = smem + L::kStageOff + warp * 2048;             // [32 heads][32 columns] BF16
    const int p_half = row / 64, p_chunk = (row % 64) / 8, p_within = (row % 8) * 2;
    int c = 0, g = 0, n_o = 0;
    bool ok = true, final_seen = false;
    float m[kHT], l[kHT];
    int unit_tiles = 0, split = 0;
    while (ok && !final_seen) {
      const int slot = c & 1;
      if (!__all_sync(0xffffffffu,
                      mbar_wait(B.tab_full + slot, (c >> 1) & 1, abort_flag, P.dev_status, P.wait_ns))) {
        ok = false;
        break;
      }
      const ChunkDesc d = desc[slot];
      mbar_arrive(B.tab_empty + slot);
      ++c;
      final_seen = (d.flags & kFlagFinal) != 0;
      if (d.flags & kFlagFirst) {
        unit_tiles = 0;
        split = d.split;
#pragma unroll
        for (int h = 0; h < kHT; ++h) {
          m[h] = head_sink[h];   // the sink seeds the max of every slice ...
          // ... and joins the denominator once (slice 0, thread 0)
          l[h] = (split == 0 && row == 0 && head_sink[h] > -INFINITY) ? 1.f : 0.f;
        }
      }
      const int ntiles = (d.nkeys + kTk - 1) / kTk;
      for (int t = 0; t < ntiles; ++t, ++g, ++unit_tiles) {
        const int sb = g & 1;
        if (!__all_sync(0xffffffffu,
                        mbar_wait(B.s_full + sb, (g >> 1) & 1, abort_flag, P.dev_status, P.wait_ns))) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        uint32_t s[32];
        tmem_ld32(lane_addr + kSCol + 32 * sb, s);
        tmem_ld_wait(s);
        tc_fence_before_sync();
        mbar_arrive(B.s_free + sb);
        const int nv = min(kTk, d.nkeys - t * kTk);
        const bool key_ok = row < nv;
        float p[kHT];
        bool flag = false;
#pragma unroll
        for (int h = 0; h < kHT; ++h) {
          const bool use = key_ok && h < heads_here;
          p[h] = use ? exp2_approx(fmaf(__uint_as_float(s[h]), P.scale_log2, -m[h])) : 0.f;
          flag |= use && !(p[h] <= kSpecBound);
        }
        // tile maxima only when some P left the bound (or a max was -inf).
        // The vote: word g%3 collects the flags of tile g before the barrier
        // and is read after it; thread 0 then clears word (g+2)%3, whose
        // last readers (tile g-1) have all passed this barrier and whose next
        // writers (tile g+2) cannot start before thread 0 reaches the next one.
        volatile uint32_t* vote = reinterpret_cast<volatile uint32_t*>(smem + L::kMiscOff + 16);
        if (__any_sync(0xffffffffu, flag) && lane == 0) atomicOr(const_cast<uint32_t*>(vote) + g % 3, 1u);
        if (!ss()) { ok = false; break; }
        const bool any = vote[g % 3] != 0u;
        if (row == 0) vote[(g + 2) % 3] = 0u;
        if (any) {
          float mx[kHT];
#pragma unroll
          for (int h = 0; h < kHT; ++h) {
            float v = (key_ok && h < heads_here) ? __uint_as_float(s[h]) * P.scale_log2 : -INFINITY;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
            mx[h] = v;
          }
          if (lane == 0) {
#pragma unroll
            for (int h = 0; h < kHT; ++h) tmax_w[warp * kHT + h] = mx[h];
          }
          if (!ss()) { ok = false; break; }
          bool moved = false;
          float alpha[kHT];
#pragma unroll
          for (int h = 0; h < kHT; ++h) {
            const float tm = fmaxf(fmaxf(tmax_w[h], tmax_w[kHT + h]), fmaxf(tmax_w[2 * kHT + h], tmax_w[3 * kHT + h]));
            const bool move = h < heads_here && (tm > m[h] || m[h] == -INFINITY) && tm > -INFINITY;
            alpha[h] = !move ? 1.f : (m[h] == -INFINITY ? 0.f : exp2_approx(m[h] - tm));
            moved |= move;
            l[h] *= alpha[h];
            if (move) m[h] = tm;
          }
          if (!ss()) { ok = false; break; }   // tmax_w is rewritten by the next tile
          if (unit_tiles > 0 && moved) {
            // O^T columns of the moved heads: wait for O^T of the previous
            // tile, then scale every column (alpha = 1 elsewhere)
            const int gp = g - 1;
            if (!__all_sync(0xffffffffu, mbar_wait(B.p_free + (gp & 1), (gp >> 1) & 1, abort_flag, P.dev_status,
                                                   P.wait_ns))) {
              ok = false;
              break;
            }
            tc_fence_after_sync();
#pragma unroll 1
            for (int b = 0; b < kOBlocks; ++b) {
              uint32_t o[32];
              tmem_ld32(lane_addr + kOCol + 32 * b, o);
              tmem_ld_wait(o);
#pragma unroll
              for (int h = 0; h < kHT; ++h) o[h] = __float_as_uint(__uint_as_float(o[h]) * alpha[h]);
              tmem_st32(lane_addr + kOCol + 32 * b, o);
            }
            tmem_st_wait();
          }
#pragma unroll
          for (int h = 0; h < kHT; ++h) {
            const bool use = key_ok && h < heads_here;
            p[h] = use ? exp2_approx(fmaf(__uint_as_float(s[h]), P.scale_log2, -m[h])) : 0.f;
          }
        }
#pragma unroll
        for (int h = 0; h < kHT; ++h) l[h] += p[h];
        // P^T as the K-major B operand [32 heads][128 keys]: this thread's
        // key is one BF16 column; the buffer was last read by O^T of tile g-2
        if (!__all_sync(0xffffffffu, mbar_wait(B.p_free + sb, ((g >> 1) & 1) ^ 1, abort_flag, P.dev_status,
                                               P.wait_ns))) {
          ok = false;
          break;
        }
        uint8_t* pb = pbuf0 + sb * L::kPBytes + p_half * (kHT * 128) + p_within;
#pragma unroll
        for (int h = 0; h < kHT; ++h) {
          const __nv_bfloat16 v = __float2bfloat16_rn(p[h]);
          *reinterpret_cast<__nv_bfloat16*>(pb + h * 128 + ((p_chunk ^ (h & 7)) << 4)) = v;
        }
        fence_proxy_async_smem();
        mbar_arrive(B.p_ready + sb);
      }
      if (!ok || !(d.flags & kFlagLast)) continue;

      // ---- epilogue of the unit: the row sums add up over the threads
      const bool have_o = unit_tiles > 0;
#pragma unroll
      for (int h = 0; h < kHT; ++h) red[h * kSoftThreads + row] = l[h];
      if (row == 0) {
#pragma unroll
        for (int h = 0; h < kHT; ++h) head_m[h] = m[h];
      }
      if (!ss()) { ok = false; break; }
      {
        const int h = row / 4, q4 = row % 4;
        float sum = 0.f;
#pragma unroll 8
        for (int k = 0; k < 32; ++k) sum += red[h * kSoftThreads + q4 * 32 + k];
        sum += __shfl_xor_sync(0xffffffffu, sum, 1);
        sum += __shfl_xor_sync(0xffffffffu, sum, 2);
        if (q4 == 0) {
          const float mh = head_m[h];
          if (S == 1) {
            head_x[h] = sum > 0.f ? 1.f / sum : 0.f;
            if (h < heads_here)
              P.lse[static_cast<int64_t>(d.i) * P.num_heads + head0 + h] =
                  sum > 0.f ? (mh + log2_approx(sum)) * kLn2 : -INFINITY;
          } else {
            reinterpret_cast<float2*>(smem + L::kMlOff)[h] = make_float2(mh, sum);
          }
        }
      }
      if (have_o) {
        if (!__all_sync(0xffffffffu, mbar_wait(B.o_done, n_o & 1, abort_flag, P.dev_status, P.wait_ns))) {
          ok = false;
          break;
        }
        ++n_o;
        tc_fence_after_sync();
      }
      if (S > 1) {   // O^T stays in TMEM for the cluster merge at the end
        if (row == 0) *reinterpret_cast<int*>(smem + L::kMiscOff + 8) = have_o ? 1 : 0;
        continue;
      }
      if (!ss()) { ok = false; break; }   // head_x is in place
      float inv[kHT];
#pragma unroll
      for (int h = 0; h < kHT; ++h) inv[h] = head_x[h];
      uint16_t* obase = P.out + (static_cast<int64_t>(d.i) * P.num_heads + head0) * kD;
#pragma unroll 1
      for (int b = 0; b < kOBlocks; ++b) {
        uint32_t o[32];
        if (have_o) {
          tmem_ld32(lane_addr + kOCol + 32 * b, o);
          tmem_ld_wait(o);
        } else {
#pragma unroll
          for (int h = 0; h < kHT; ++h) o[h] = 0u;
        }
        // transpose through the warp's stage: column `lane` of each head row
#pragma unroll
        for (int h = 0; h < kHT; ++h)
          reinterpret_cast<__nv_bfloat16*>(stage + h * 64)[lane] = __float2bfloat16_rn(__uint_as_float(o[h]) * inv[h]);
        __syncwarp();
#pragma unroll
        for (int k = 0; k < 4; ++k) {   // 8 head rows x 64 bytes per instruction
          const int h = 8 * k + (lane >> 2), pc = lane & 3;
          const uint4 v = *reinterpret_cast<const uint4*>(stage + h * 64 + pc * 16);
          if (h < heads_here)
            *reinterpret_cast<uint4*>(obase + static_cast<int64_t>(h) * kD + 128 * b + warp * 32 + pc * 8) = v;
        }
        __syncwarp();
      }
      tc_fence_before_sync();
      if (have_o) mbar_arrive(B.o_free);   // one phase per unit with O^T products, as the MMA waits
      if (!ss()) { ok = false; break; }   // red, head_x are reused by the next unit
    }
    cta_finish(P, true, smem, sbase, tmem, tid, warp, head0, heads_here, &ss);
  }
}

}  // namespace

int d512_default_splits(int32_t n_queries, int32_t num_heads) {
  const int64_t units = static_cast<int64_t>(n_queries) * ((num_heads + kHT - 1) / kHT);
  const int64_t sms = device_sm_count();
  if (units <= 0 || units >= sms) return 1;
  int64_t s = sms / units;
  s = s >= 8 ? 8 : (s >= 4 ? 4 : (s >= 2 ? 2 : 1));   // slices that divide the 512 columns evenly
  return static_cast<int>(s);
}

cudaError_t launch_sparse_sink_attn_d512(const AttnArgs& a, cudaStream_t stream) {
  if (a.n_queries == 0) return cudaSuccess;
  Params P;
  memset(&P, 0, sizeof P);
  if (tensor_map_encoder() == nullptr) return cudaErrorNotSupported;
  P.q_box_rows = a.num_heads < kHT ? a.num_heads : kHT;
  {
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kD), static_cast<cuuint64_t>(a.num_heads),
                                static_cast<cuuint64_t>(a.n_queries)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(a.q_stride_head) * 2,
                                   static_cast<cuuint64_t>(a.q_stride_tok) * 2};
    const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(P.q_box_rows), 1};
    const cuuint32_t elem[3] = {1, 1, 1};
    if (tensor_map_encoder()(&P.tm_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<uint16_t*>(a.q), dims, strides,
                             box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  P.k_raw = reinterpret_cast<const uint8_t*>(a.k_raw);
  P.v_raw = reinterpret_cast<const uint8_t*>(a.v_raw);
  P.k_cmp = reinterpret_cast<const uint8_t*>(a.k_cmp);
  P.v_cmp = reinterpret_cast<const uint8_t*>(a.v_cmp);
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
  P.scale_log2 = static_cast<float>(static_cast<double>(a.scale) * 1.4426950408889634);
  P.out = a.out;
  P.lse = a.lse;
  P.num_splits = a.num_splits;
  P.dev_status = a.dev_status;
  P.wait_ns = attn_wait_limit_ns();
  P.stall = attn_stall() ? 1 : 0;
  static bool configured = false;
  if (!configured) {
    cudaError_t err = cudaFuncSetAttribute(sparse_sink_attn_d512_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           Layout::kBytes);
    if (err != cudaSuccess) return err;
    configured = true;
  }
  const int head_tiles = (a.num_heads + kHT - 1) / kHT;
  const int64_t units = static_cast<int64_t>(a.n_queries) * a.num_splits;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = Layout::kBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // may start early
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (a.num_splits > 1) {
    // one unit per CTA, the slices of a query in one cluster
    cfg.gridDim = dim3(static_cast<unsigned>(units), head_tiles);
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = static_cast<unsigned>(a.num_splits);
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.numAttrs = 2;
  } else {
    // persistent: one CTA per SM, units strided over the CTAs
    const int64_t slots = std::max<int64_t>(1, static_cast<int64_t>(device_sm_count()) / head_tiles);
    cfg.gridDim = dim3(static_cast<unsigned>(std::min<int64_t>(units, slots)), head_tiles);
  }
  cudaError_t err = cudaLaunchKernelEx(&cfg, sparse_sink_attn_d512_kernel, P);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

}  // namespace spa
