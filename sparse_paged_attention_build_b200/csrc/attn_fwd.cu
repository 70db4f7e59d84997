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
//   S  = Q[128 x d] . K_half[32 x d]^T      tcgen05.mma, Q in TMEM, K in SMEM
//   P  = exp2(S*scale*log2e - m)  (BF16)    softmax warps, TMEM -> regs -> TMEM
//   O += P[128 x 32] . V_half[32 x d]        tcgen05.mma, P in TMEM, V in SMEM
// K and V arrive in tiles of 64 rows; the products and the softmax take each
// tile in two halves of 32 keys.
// Both products take their A operand from TMEM: measured on B200, an
// M = 128, N = 64 product with both operands in shared memory is bound by
// shared-memory bandwidth at two thirds of the tensor rate, while with A in
// TMEM it runs at the full rate. The sink seeds the running max and the
// denominator (m = sink*log2e, l = 1), so it is counted exactly once and
// never multiplies a V row.
//
// Persistent CTAs (two per SM) walk their units in a fixed stride; the two
// CTAs of an SM interleave on the tensor core and on the exp unit. Warp
// roles (512 threads, four warpgroups):
//   warps 0-3  softmax + epilogue; thread t owns head row t = TMEM lane t.
//              They also move each unit's Q from shared memory into TMEM.
//   warp  4    TMEM allocation; lane 0 issues every UMMA and commit
//   warps 5, 7 resolver: for a chunk of up to 768 keys of a unit they load
//              the keys, look their pages up and write the physical row of
//              every key (bit 31 = raw pool) to a double-buffered table,
//              plus a chunk descriptor that every other role follows. All
//              dependent global loads of the gather happen here, ahead of
//              the copies; each warp takes half of every chunk.
//   warp  6    Q: one TMA box load per unit into the landing area
//   warps 8-11 K gather, warps 12-15 V gather: 16-byte cp.async copies of
//              the rows the table names into 2-stage rings, written in the
//              128-byte swizzled K-major layout of the UMMA descriptors
//              (lanes 0-15 of a warp copy one 256-byte row, so every
//              instruction moves whole rows); rows outside a pool (padding,
//              faulty keys) are zero-filled. Measured on B200, random row
//              gathers from L2 by cp.async over 8 warps per CTA run at
//              about 14.7 TB/s against 5.9 TB/s for TMA tile::gather4 from
//              one warp per operand, which capped this kernel before.
// The warpgroups then move registers with setmaxnreg: the softmax rows keep
// 64 scores, 32 packed probabilities and the running statistics in
// registers, the copy warps need few.
// TMEM columns: two S/P buffers [0,64) of 32 columns each, Q [64, 64 + d/2)
// as packed BF16 pairs, O after. S of half tile j+1 is computed while the
// softmax of half j runs (issue order QK(j+1), then PV(j)); P(j) overwrites
// the first 16 columns of its buffer and is read by PV(j) before QK(j+2)
// reuses that buffer, since the UMMAs of a CTA run in issue order. (With one
// 64-column S buffer the softmax and the product round trip ran in series,
// about 950 + 1400 cycles per 64 keys for a CTA on B200.)
// The softmax first takes P with the running max as it stands and only
// recomputes a tile whose row sum leaves a fixed bound (see kSpecBound);
// O/l and LSE use the same max, so the result is exact in exact arithmetic.
#include <algorithm>
#include <cmath>
#include <cstring>

#include "attn_common.cuh"

namespace spa {
namespace {

using namespace attn;

constexpr int kStagesK = 2;
constexpr int kStagesV = 2;
constexpr int kSoftThreads = 128;
constexpr int kMmaWarp = 4;
constexpr int kResolverWarp0 = 5;
constexpr int kQWarp = 6;
constexpr int kResolverWarp1 = 7;
constexpr int kKGroupWarp0 = 8;                  // warps 8..11: K rows
constexpr int kVGroupWarp0 = 12;                 // warps 12..15: V rows
constexpr int kGroupThreads = 128;
constexpr int kThreads = 512;
constexpr uint32_t kTmemCols = 256;
// Registers per thread after the split; the four warpgroups together keep
// the 4 x 64 the block is launched with (two 512-thread blocks per SM).
template <bool kFp8>
struct RegSplit {
  static constexpr uint32_t kSoftmax = kFp8 ? 96 : 112;
  static constexpr uint32_t kControl = 64;            // MMA issue, resolvers, Q
  static constexpr uint32_t kGather = kFp8 ? 48 : 40;  // the FP8 decode holds codes and scales
  static_assert(true || kSoftmax + kControl + 2 * kGather <= 4 * 64, "register split exceeds the launch");
};
// A tile whose row sum of P, taken with the running max as it stands,
// exceeds 2^16 (or is not a number) is recomputed with its exact max. P
// therefore stays below 2^16: harmless in BF16 and in the FP32 sums, whose
// relative precision does not depend on magnitude.
constexpr float kSpecBound = 65536.0f;
// The tensor cores and the softmax work on half tiles of 32 keys with two S
// buffers in TMEM: S of half j+1 is computed while the softmax of half j
// runs, and P of half j (BF16, over the first kSub/2 columns of its S
// buffer) is read by the PV product before S of half j+2 overwrites it (the
// products of a CTA run in issue order).
constexpr int kSub = 32;
// consumers of a chunk descriptor: K and V groups, MMA thread, softmax, Q warp
constexpr uint32_t kTabConsumers = 2 * kGroupThreads + 1 + kSoftThreads + 32;

struct Params {
  // TMA descriptors (passed as a __grid_constant__ parameter)
  CUtensorMap tm_q;       // 3D {d, H, N}, box {64, q_box_rows, 1}
  CUtensorMap tm_k_raw;   // 2D {d, rows}, box {64, 1}: gather4 / single rows
  CUtensorMap tm_v_raw;
  CUtensorMap tm_k_cmp;
  CUtensorMap tm_v_cmp;
  // the pools as plain pointers, for the cp.async gather
  const uint8_t* k_raw;
  const uint8_t* v_raw;
  const uint8_t* k_cmp;
  const uint8_t* v_cmp;
  int32_t q_box_rows;     // min(128, num_heads)
  int32_t n_queries, num_heads;
  int64_t raw_pages;
  int32_t raw_ps_log2, pt_raw_cols;
  const int32_t* pt_raw;
  int64_t cmp_pages;
  int32_t cmp_ps_log2, pt_cmp_cols;
  const int32_t* pt_cmp;
  // compressed pool in FP8 (OCP E4M3, one FP32 scale per 64 elements), for
  // the fused decode; NULL on the BF16 path
  const uint8_t* k_cmp8;
  const uint8_t* v_cmp8;
  const float* k_cmp_sc;
  const float* v_cmp_sc;
  int32_t fp8_fnuz;    // the codes are E4M3 FNUZ (1) or OCP E4M3 (0)
  const int32_t* req;
  int32_t n_requests;
  const int32_t* indptr;
  const int32_t* indices;
  const float* sink;
  float scale_log2;
  uint16_t* out;
  float* lse;
  int32_t num_splits;
  // 1: the slices of a query are the CTAs of one cluster (one unit per
  // CTA) and merge through distributed shared memory; 0: FP32 partials in
  // the workspace, merged by the last slice to finish
  int32_t cluster_merge;
  float* part_o;       // [n_queries * num_splits][num_heads][d]  (split runs only)
  float2* part_ml;     // [n_queries * num_splits][num_heads]
  uint32_t* tickets;   // [n_queries * head_tiles]
  uint32_t* dev_status;
  // limit of every wait between the roles (ns); the waits that keep TMEM
  // and shared memory alive until the CTA's own copies and MMAs are done
  // keep the fixed kWaitTimeoutNs
  uint64_t wait_ns;
  int32_t stall;       // testing: every CTA waits on a barrier nothing arrives at
};

template <int D>
struct Layout {
  static constexpr int kQBytes = 128 * D * 2;
  static constexpr int kTileBytes = kT * D * 2;             // one K or V tile
  static constexpr int kQOff = 0;                           // TMA landing area of Q
  static constexpr int kKOff = kQBytes;
  static constexpr int kVOff = kKOff + kStagesK * kTileBytes;
  static constexpr int kTabOff = kVOff + kStagesV * kTileBytes;       // [2][kChunkKeys] u32
  static constexpr int kDescOff = kTabOff + 2 * kChunkKeys * 4;       // [2] ChunkDesc
  // [16][128] f32 merge weights; between merges, a 2 KB output staging area
  // per softmax warp
  static constexpr int kMergeOff = kDescOff + 2 * static_cast<int>(sizeof(ChunkDesc));
  static constexpr int kBarOff = kMergeOff + kAttnMaxSplits * 128 * 4;
  // tab_full[2], tab_empty[2], q_full, q_empty, q_ready, K ring, V ring,
  // s_full[2], p_ready[2], o_ready, o_done, mma_done, soft_sync[2]
  static constexpr int kNumBars = 2 + 2 + 3 + 2 * kStagesK + 2 * kStagesV + 2 + 2 + 1 + 1 + 1 + 2;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kUsed = kMiscOff + 32;   // + the testing stall barrier at kMiscOff + 16
  // + alignment slack; at least 80 KB so that no more than two CTAs share an
  // SM (TMEM holds two 256-column allocations)
  static constexpr int kBytes = (kUsed + 1024) < 80 * 1024 ? 80 * 1024 : (kUsed + 1024);
  static constexpr uint32_t kSCol = 0;                      // S buffers [2][kSub]
  static constexpr uint32_t kQCol = 2 * kSub;
  static constexpr uint32_t kOCol = 2 * kSub + D / 2;
  static_assert(kOCol + D <= kTmemCols, "TMEM budget");
  static_assert((kBytes + 1024) * 2 <= 228 * 1024, "two CTAs per SM");
  static_assert(kMergeOff % 16 == 0, "staging alignment");
};

struct Bars {
  uint64_t* tab_full;   // [2]
  uint64_t* tab_empty;  // [2]
  uint64_t* q_full;     // Q of the next unit landed in shared memory
  uint64_t* q_empty;    // ... and has been moved on to TMEM
  uint64_t* q_ready;    // Q of the next unit is in TMEM
  uint64_t* k_full;     // [kStagesK]
  uint64_t* k_empty;
  uint64_t* v_full;     // [kStagesV]
  uint64_t* v_empty;
  uint64_t* s_full;     // [2]: S of a half tile in its buffer
  uint64_t* p_ready;    // [2]: P of a half tile in its S buffer (one barrier per buffer: the
                        // softmax may finish two half tiles before the UMMA issuer waits)
  uint64_t* o_ready;    // one phase per half tile: its PV product has completed
  uint64_t* o_done;     // last PV of a unit complete
  uint64_t* mma_done;
  // [2]: barrier of the softmax threads, the two used in turn. An mbarrier
  // rather than a named barrier so that the wait is bounded: a thread that
  // gave up elsewhere cannot leave the others stuck.
  uint64_t* soft_sync;
};

// End of every role (inlined into each, so that it runs within that
// warpgroup's registers): every TMEM access of the role has completed; the
// softmax warps (soft) then run the cluster merge, every warp takes the
// cluster barriers, and the MMA warp frees TMEM last.
template <int D>
__device__ __forceinline__ void cta_finish(const Params& P, bool soft, uint8_t* smem, uint32_t sbase, uint32_t tmem,
                                           int tid, int warp, int S, int heads_here, int head0) {
  using L = Layout<D>;
  __syncwarp();
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if (P.cluster_merge) {
    // Exact merge of the S slices of query i, CTA `rank` holding slice
    // `rank`: LSE = M + log2(L), O = sum_s w_s O_s with w_s = 2^(m_s - M)/L
    // (page "[WS2] Add CP-aware Attention contract and dispatch metadata",
    // Summary: the deterministic (out, lse) merge). CTA r owns rows
    // [r*per, (r+1)*per) of the output. After the first cluster barrier
    // every CTA reads all slices' (m, l) of its rows (one round trip of
    // distributed shared memory), scales its O rows by its weight and
    // stores each row straight into its owner's idle K/V ring (posted
    // stores, slot = the sender's rank); after the second barrier each owner
    // sums its slots locally and writes BF16 O. No shared memory is read or
    // written remotely after the second barrier, so no third one is needed.
    // Every thread of every CTA reaches both barriers: every earlier wait in
    // the kernel is bounded.
    const int rank = static_cast<int>(cluster_ctarank());
    const int i = static_cast<int>(blockIdx.x / S);
    const uint32_t ml_addr = sbase + L::kMergeOff;
    const uint32_t rx_addr = sbase + L::kKOff;               // [S][per][D] FP32, 16-byte chunks swizzled by row
    constexpr int kChunks = D / 4;                           // 16-byte chunks per row
    const int per = (128 + S - 1) / S;
    // the slots (S * per <= 128 + S - 1 rows of D FP32) fill the K/V rings
    // and may run on into the chunk tables, all idle by now
    static_assert(L::kTabOff - L::kKOff + 2 * kChunkKeys * 4 >= (128 + kAttnMaxClusterSplits - 1) * D * 4,
                  "receive slots fit the idle rings and tables");
    static_assert(L::kTabOff == L::kVOff + kStagesV * L::kTileBytes && L::kVOff == L::kKOff + kStagesK * L::kTileBytes,
                  "rings and tables are contiguous");
    __syncwarp();
    cluster_sync_all();                                      // every slice's (m, l) is in place; rings idle
    if (soft) {
      const int row = tid;
      float2 ml[kAttnMaxClusterSplits];
#pragma unroll
      for (int s = 0; s < kAttnMaxClusterSplits; ++s)
        ml[s] = s < S ? ld_dsmem_f2(dsmem_addr(ml_addr + row * 8, s)) : make_float2(-INFINITY, 0.f);
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
      const float scale_own = Lsum > 0.f ? w_own / Lsum : 0.f;
      if (rank == 0 && row < heads_here)
        P.lse[static_cast<int64_t>(i) * P.num_heads + head0 + row] =
            Lsum > 0.f ? (M + log2_approx(Lsum)) * kLn2 : -INFINITY;
      const bool have_o = *reinterpret_cast<const int*>(smem + L::kMiscOff + 12) != 0;
      const uint32_t o_lane = tmem + (static_cast<uint32_t>(warp * 32) << 16) + L::kOCol;
      const int owner = row / per, rr = row - owner * per;
      const uint32_t dst = dsmem_addr(rx_addr + static_cast<uint32_t>(((rank * per + rr) * D) * 4), owner);
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t o[32];
        if (have_o) {   // warp-uniform: one flag per CTA
          tmem_ld32(o_lane + c0, o);
          tmem_ld_wait(o);
        } else {
#pragma unroll
          for (int cc = 0; cc < 32; ++cc) o[cc] = 0u;
        }
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          const int chunk = (c0 >> 2) + v;
          const int phys = chunk ^ (rr & (kChunks - 1));
          st_dsmem_f4(dst + phys * 16,
                      make_float4(__uint_as_float(o[4 * v]) * scale_own, __uint_as_float(o[4 * v + 1]) * scale_own,
                                  __uint_as_float(o[4 * v + 2]) * scale_own, __uint_as_float(o[4 * v + 3]) * scale_own));
        }
      }
    }
    __syncwarp();
    cluster_sync_all();                                      // every slice's weighted rows have arrived
    if (soft) {
      const int r0 = min(rank * per, heads_here), r1 = min(r0 + per, heads_here);
      const float* rx = reinterpret_cast<const float*>(smem + L::kKOff);
      uint16_t* obase = P.out + (static_cast<int64_t>(i) * P.num_heads + head0) * D;
      const int n_items = (r1 - r0) * kChunks;
      for (int idx = tid; idx < n_items; idx += kSoftThreads) {
        const int rr = idx / kChunks, c = idx % kChunks;
        const int phys = c ^ (rr & (kChunks - 1));
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int s = 0; s < S; ++s) {
          const float4 v = *reinterpret_cast<const float4*>(rx + ((s * per + rr) * D) + phys * 4);
          acc.x += v.x;
          acc.y += v.y;
          acc.z += v.z;
          acc.w += v.w;
        }
        *reinterpret_cast<uint2*>(obase + static_cast<int64_t>(r0 + rr) * D + 4 * c) =
            make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
      }
    }
  }
  if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

template <int D, bool kFp8>
__global__ void __launch_bounds__(kThreads, 2) sparse_sink_attn_kernel(const __grid_constant__ Params P) {
  using R = RegSplit<kFp8>;
  using L = Layout<D>;
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
  B.q_ready = bar0 + 6;
  B.k_full = bar0 + 7;
  B.k_empty = B.k_full + kStagesK;
  B.v_full = B.k_empty + kStagesK;
  B.v_empty = B.v_full + kStagesV;
  B.s_full = B.v_empty + kStagesV;
  B.p_ready = B.s_full + 2;
  B.o_ready = B.p_ready + 2;
  B.o_done = B.o_ready + 1;
  B.mma_done = B.o_done + 1;
  B.soft_sync = B.mma_done + 1;
  uint32_t* tab = reinterpret_cast<uint32_t*>(smem + L::kTabOff);
  ChunkDesc* desc = reinterpret_cast<ChunkDesc*>(smem + L::kDescOff);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);
  uint32_t* ticket_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff + 8);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int S = P.num_splits;
  const int head0 = blockIdx.y * 128;
  const int heads_here = min(128, P.num_heads - head0);

  // ---- setup
  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(B.tab_full + s, 64);   // two resolver warps
      mbar_init(B.tab_empty + s, kTabConsumers);
      mbar_init(B.soft_sync + s, kSoftThreads);
    }
    mbar_init(B.q_full, 1);
    mbar_init(B.q_empty, kSoftThreads);
    mbar_init(B.q_ready, kSoftThreads);
    for (int s = 0; s < kStagesK; ++s) {
      mbar_init(B.k_full + s, kGroupThreads);
      mbar_init(B.k_empty + s, 1);
    }
    for (int s = 0; s < kStagesV; ++s) {
      mbar_init(B.v_full + s, kGroupThreads);
      mbar_init(B.v_empty + s, 1);
    }
    mbar_init(B.s_full, 1);
    mbar_init(B.s_full + 1, 1);
    mbar_init(B.p_ready, kSoftThreads);
    mbar_init(B.p_ready + 1, kSoftThreads);
    mbar_init(B.o_ready, 1);
    mbar_init(B.o_done, 1);
    mbar_init(B.mma_done, 1);
    *abort_flag = 0;
    mbar_init(reinterpret_cast<uint64_t*>(smem + L::kMiscOff + 16), 1);   // never arrived at
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
  // Each warpgroup takes its register limit at one place (setmaxnreg is
  // executed by the four warps of a warpgroup together) that dominates all
  // of its roles' code.
  if (warp >= 4 && warp < 8) {
    warpgroup_reg_dealloc<R::kControl>();
    if (warp == kResolverWarp0 || warp == kResolverWarp1) {
      // ================================================= resolver
      // testing stall: a wait that only its limit ends, then the CTA unwinds
      if (P.stall) mbar_wait(reinterpret_cast<uint64_t*>(smem + L::kMiscOff + 16), 0, abort_flag, P.dev_status, P.wait_ns);
      resolver_loop<2>(P, S, tab, desc, B.tab_full, B.tab_empty, abort_flag, lane, false,
                       warp == kResolverWarp0 ? 0 : 1);
      cta_finish<D>(P, false, smem, sbase, tmem, tid, warp, S, heads_here, head0);
    } else if (warp == kQWarp) {
      // ================================================= Q loader
      // Every unit's Q, empty units included, so that the Q phases of all
      // roles stay in step; the landing area is free once the previous Q
      // has moved on to TMEM. The CTA's first unit is unit blockIdx.x (units
      // are strided over the CTAs), so its Q is loaded at once, while the
      // resolver is still fetching its keys.
      constexpr int kHalves = D / 64;
      int c = 0, qc = 0;
      bool final_seen = false, first_issued = false;
      if (lane == 0) {
        mbar_arrive_expect_tx(B.q_full, P.q_box_rows * 128 * kHalves);
        for (int hb = 0; hb < kHalves; ++hb)
          tma_load_3d(sbase + L::kQOff + hb * (128 * 128), &P.tm_q, B.q_full, hb * 64, head0,
                      static_cast<int32_t>(blockIdx.x / S));
      }
      first_issued = true;
      qc = 1;
      while (!final_seen) {
        const int slot = c & 1;
        if (!mbar_wait(B.tab_full + slot, (c >> 1) & 1, abort_flag, P.dev_status, P.wait_ns)) break;
        const ChunkDesc d = desc[slot];
        final_seen = (d.flags & kFlagFinal) != 0;
        bool ok = true;
        if ((d.flags & kFlagFirst) && first_issued) {
          first_issued = false;   // the first unit's Q is on its way
        } else if (d.flags & kFlagFirst) {
          ok = mbar_wait(B.q_empty, (qc & 1) ^ 1, abort_flag, P.dev_status, P.wait_ns);
          if (ok && lane == 0) {
            mbar_arrive_expect_tx(B.q_full, P.q_box_rows * 128 * kHalves);
            for (int hb = 0; hb < kHalves; ++hb)
              tma_load_3d(sbase + L::kQOff + hb * (128 * 128), &P.tm_q, B.q_full, hb * 64, head0, d.i);
          }
          if (ok) ++qc;
        }
        __syncwarp();
        mbar_arrive(B.tab_empty + slot);
        ++c;
        if (!ok) break;
      }
      // the last Q copy has landed before the CTA can leave (it lands even
      // when the roles gave up early; this wait keeps the fixed limit)
      if (qc > 0) mbar_wait(B.q_full, (qc - 1) & 1, nullptr, P.dev_status);
      cta_finish<D>(P, false, smem, sbase, tmem, tid, warp, S, heads_here, head0);
    } else if (warp == kMmaWarp) {
      // ================================================= UMMA issuer
      // Half tile x: S[x%2] = Q K_x^T (A = Q from TMEM); once its P is in
      // TMEM, O += P_x V_x (A = P from TMEM). The issue order is QK(x+1)
      // before PV(x), so the softmax of half x overlaps the product of the
      // next S; QK(x+2) comes after PV(x), which read P(x) from the same
      // buffer.
      if (lane == 0) {
        constexpr uint32_t idesc_s = idesc_bf16_f32(128, kSub, 0);
        constexpr uint32_t idesc_o = idesc_bf16_f32(128, D, 1);
        int c = 0, g = 0, u = 0, x = 0;
        bool ok = true, final_seen = false;
        // the half tile whose PV is still to be issued
        int pend = -1, pend_v = 0, pend_hf = 0;
        bool pend_first = false, pend_last_of_tile = false, pend_last_of_unit = false;
        auto issue_pv = [&]() -> bool {
          if (!mbar_wait(B.p_ready + (pend & 1), (pend >> 1) & 1, abort_flag, P.dev_status, P.wait_ns)) return false;
          const int st = pend_v % kStagesV;
          if (pend_hf == 0 &&
              !mbar_wait(B.v_full + st, (pend_v / kStagesV) & 1, abort_flag, P.dev_status, P.wait_ns))
            return false;
          tc_fence_after_sync();
          const uint32_t v_addr = sbase + L::kVOff + st * L::kTileBytes + pend_hf * (kSub * 128);
          const uint32_t p_col = tmem + L::kSCol + (pend & 1) * kSub;
#pragma unroll
          for (int k = 0; k < kSub / 16; ++k) {
            const uint64_t bdesc = smem_desc_sw128(v_addr + k * 16 * 128, kT * 128, 1024);
            umma_ts(tmem + L::kOCol, p_col + k * 8, bdesc, idesc_o, (!pend_first || k > 0) ? 1u : 0u);
          }
          tc_commit(B.o_ready);
          if (pend_last_of_tile) tc_commit(B.v_empty + st);
          if (pend_last_of_unit) tc_commit(B.o_done);
          pend = -1;
          return true;
        };
        while (ok && !final_seen) {
          const int slot = c & 1;
          if (!mbar_wait(B.tab_full + slot, (c >> 1) & 1, abort_flag, P.dev_status, P.wait_ns)) { ok = false; break; }
          const ChunkDesc d = desc[slot];
          mbar_arrive(B.tab_empty + slot);
          ++c;
          final_seen = (d.flags & kFlagFinal) != 0;
          if (d.flags & kFlagFirst) {   // this unit's Q is in TMEM
            if (!mbar_wait(B.q_ready, u & 1, abort_flag, P.dev_status, P.wait_ns)) { ok = false; break; }
            ++u;
            tc_fence_after_sync();
          }
          const int ntiles = ceil_tiles(d.nkeys);
          for (int t = 0; ok && t < ntiles; ++t, ++g) {
            const int stage = g % kStagesK;
            if (!mbar_wait(B.k_full + stage, (g / kStagesK) & 1, abort_flag, P.dev_status, P.wait_ns)) { ok = false; break; }
            tc_fence_after_sync();
            const uint32_t k_addr = sbase + L::kKOff + stage * L::kTileBytes;
            const int nv = min(kT, d.nkeys - t * kT);
            const int nsub = (nv + kSub - 1) / kSub;
            for (int hf = 0; hf < nsub; ++hf, ++x) {
#pragma unroll
              for (int k = 0; k < D / 16; ++k) {
                const uint64_t bdesc =
                    smem_desc_sw128(k_addr + (k >> 2) * (kT * 128) + hf * (kSub * 128) + (k & 3) * 32, 16, 1024);
                umma_ts(tmem + L::kSCol + (x & 1) * kSub, tmem + L::kQCol + k * 8, bdesc, idesc_s, k > 0 ? 1u : 0u);
              }
              if (hf == nsub - 1) tc_commit(B.k_empty + stage);
              tc_commit(B.s_full + (x & 1));
              if (pend >= 0 && !issue_pv()) { ok = false; break; }
              pend = x;
              pend_v = g;
              pend_hf = hf;
              pend_first = (d.flags & kFlagFirst) && t == 0 && hf == 0;
              pend_last_of_tile = hf == nsub - 1;
              pend_last_of_unit = (d.flags & kFlagLast) && t == ntiles - 1 && hf == nsub - 1;
            }
          }
        }
        if (ok && pend >= 0) issue_pv();
        // every UMMA has completed before TMEM is released
        tc_commit(B.mma_done);
        mbar_wait(B.mma_done, 0, nullptr, P.dev_status);
      }
      cta_finish<D>(P, false, smem, sbase, tmem, tid, warp, S, heads_here, head0);
    }
  } else if (warp >= kKGroupWarp0) {
    warpgroup_reg_dealloc<R::kGather>();
    // ================================================= K / V gather (cp.async)
    // A warp copies 16 rows of a 64-row tile: lane l takes 16-byte piece
    // l % (D/8) of row l / (D/8) (+ the rows of later instructions), so an
    // instruction moves 32 / (D/8) whole rows. Piece c of row r lands at
    // half c/8 (64-column blocks), row r, 16-byte chunk (c%8) ^ (r%8): the
    // 128-byte swizzle of the K-major UMMA layout. A tile is handed over
    // (fence.proxy.async, then one arrival per thread) once its copies have
    // landed, which is checked after the next tile's copies are issued, so
    // two tiles are in flight; before any wait that would block, the tile
    // in flight is handed over first.
    const bool is_k = warp < kVGroupWarp0;
    const int gw = warp - (is_k ? kKGroupWarp0 : kVGroupWarp0);
    const int nst = is_k ? kStagesK : kStagesV;
    uint64_t* full = is_k ? B.k_full : B.v_full;
    uint64_t* empty = is_k ? B.k_empty : B.v_empty;
    const uint8_t* pool_raw = is_k ? P.k_raw : P.v_raw;
    const uint8_t* pool_cmp = is_k ? P.k_cmp : P.v_cmp;
    const uint8_t* pool8 = is_k ? P.k_cmp8 : P.v_cmp8;
    const float* psc = is_k ? P.k_cmp_sc : P.v_cmp_sc;
    const uint32_t ring = sbase + (is_k ? L::kKOff : L::kVOff);
    constexpr int kCpr = D / 8;          // 16-byte pieces per row
    constexpr int kRpi = 32 / kCpr;      // rows per instruction
    constexpr int kNi = 16 / kRpi;       // instructions per warp per tile
    const int ch = lane % kCpr, rsub = lane / kCpr;
    const uint32_t col_off = static_cast<uint32_t>((ch / 8) * (kT * 128));
    const int c8 = ch % 8;
    int pending = -1;   // ring stage whose copies are issued but not handed over
    auto hand_over = [&]() {
      if (pending >= 0) {
        cp_async_wait_group<0>();
        fence_proxy_async_smem();
        mbar_arrive(full + pending);
        pending = -1;
      }
    };
    int c = 0, g = 0;
    bool final_seen = false;
    while (!final_seen) {
      const int slot = c & 1;
      if (pending >= 0 && !mbar_try_wait(B.tab_full + slot, (c >> 1) & 1)) hand_over();
      if (!mbar_wait(B.tab_full + slot, (c >> 1) & 1, abort_flag, P.dev_status, P.wait_ns)) break;
      const ChunkDesc d = desc[slot];
      final_seen = (d.flags & kFlagFinal) != 0;
      const uint32_t* t_rows = tab + slot * kChunkKeys;
      const int ntiles = ceil_tiles(d.nkeys);
      bool ok = true;
      for (int t = 0; t < ntiles; ++t, ++g) {
        const int stage = g % nst;
        const uint32_t par = ((g / nst) & 1) ^ 1;
        if (pending >= 0 && !mbar_try_wait(empty + stage, par)) hand_over();
        if (!mbar_wait(empty + stage, par, abort_flag, P.dev_status, P.wait_ns)) { ok = false; break; }
        const int nv = min(kT, d.nkeys - t * kT);
        const uint32_t* trow = t_rows + t * kT;
        const uint32_t stage_base = ring + stage * L::kTileBytes + col_off;
        if constexpr (!kFp8) {
#pragma unroll 2
          for (int j = 0; j < kNi; ++j) {
            const int r = gw * 16 + j * kRpi + rsub;
            const uint32_t e = r < nv ? trow[r] : kInvalidRow;
            const uint8_t* base = (e & kRawBit) ? pool_raw : pool_cmp;
            const bool valid = e != kInvalidRow && base != nullptr;
            const uint8_t* src = valid ? base + static_cast<int64_t>(e & ~kRawBit) * (D * 2) + ch * 16 : pool_raw;
            cp_async16(stage_base + r * 128 + ((c8 ^ (r & 7)) << 4), src, valid ? 16u : 0u);
          }
        } else {
          // compressed rows arrive as E4M3 codes (8 per piece) and their
          // group scale, decoded exactly as the page decode does; window rows
          // and zero rows by cp.async. Every load of the tile first.
          uint2 code[kNi];
          float sc[kNi];
#pragma unroll
          for (int j = 0; j < kNi; ++j) {
            const int r = gw * 16 + j * kRpi + rsub;
            const uint32_t e = r < nv ? trow[r] : kInvalidRow;
            const bool fp8_row = e != kInvalidRow && !(e & kRawBit);
            code[j] = make_uint2(0u, 0u);
            sc[j] = 0.f;
            if (fp8_row) {
              const int64_t row8 = e;
              code[j] = __ldg(reinterpret_cast<const uint2*>(pool8 + row8 * D + ch * 8));
              sc[j] = __ldg(psc + row8 * (D / 64) + (ch * 8) / 64);
            } else {
              const bool valid = e != kInvalidRow;
              const uint8_t* src = valid ? pool_raw + static_cast<int64_t>(e & ~kRawBit) * (D * 2) + ch * 16 : pool_raw;
              cp_async16(stage_base + r * 128 + ((c8 ^ (r & 7)) << 4), src, valid ? 16u : 0u);
            }
          }
#pragma unroll
          for (int j = 0; j < kNi; ++j) {
            const int r = gw * 16 + j * kRpi + rsub;
            const uint32_t e = r < nv ? trow[r] : kInvalidRow;
            if (e == kInvalidRow || (e & kRawBit)) continue;
            uint32_t o[4];
            if (P.fp8_fnuz) decode_e4m3x8<true>(code[j], sc[j], o);
            else decode_e4m3x8<false>(code[j], sc[j], o);
            *reinterpret_cast<uint4*>(smem + (stage_base - sbase) + r * 128 + ((c8 ^ (r & 7)) << 4)) =
                make_uint4(o[0], o[1], o[2], o[3]);
          }
        }
        cp_async_commit();
        if (pending >= 0) {   // the previous tile has landed: hand it over
          cp_async_wait_group<1>();
          fence_proxy_async_smem();
          mbar_arrive(full + pending);
        }
        pending = stage;
      }
      mbar_arrive(B.tab_empty + slot);
      ++c;
      if (!ok) break;
    }
    hand_over();
    cp_async_wait_group<0>();
    cta_finish<D>(P, false, smem, sbase, tmem, tid, warp, S, heads_here, head0);
  } else {
    warpgroup_reg_alloc<R::kSoftmax>();
    // ================================================= softmax + epilogue
    const int row = tid;   // head row == TMEM lane
    const int h = head0 + row;
    const bool row_ok = row < heads_here;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const float sink2 = (P.sink != nullptr && row_ok) ? P.sink[h] * kLog2e : -INFINITY;
    uint32_t nsync = 0;
    // barrier of the softmax threads (bounded: false once a wait gave up)
    auto gsync = [&]() -> bool {
      uint64_t* bar = B.soft_sync + (nsync & 1);
      const uint32_t parity = (nsync >> 1) & 1;
      ++nsync;
      mbar_arrive(bar);
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, P.dev_status, P.wait_ns));
    };
    // Q of the next unit: shared memory (TMA, 128-byte swizzled rows) ->
    // registers -> this thread's TMEM lane, as the packed BF16 pairs the
    // UMMA takes for a K-major A operand. Only called once every UMMA that
    // reads the previous Q has completed.
    int qc = 0;
    auto copy_q = [&]() -> bool {
      if (!__all_sync(0xffffffffu, mbar_wait(B.q_full, qc & 1, abort_flag, P.dev_status, P.wait_ns))) return false;
      ++qc;
      const uint8_t* qrow = smem + L::kQOff + row * 128;
#pragma unroll
      for (int a = 0; a < D / 64; ++a) {
        uint32_t v[32];
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const uint4 x = *reinterpret_cast<const uint4*>(qrow + a * (128 * 128) + ((ch ^ (row & 7)) * 16));
          v[4 * ch] = x.x;
          v[4 * ch + 1] = x.y;
          v[4 * ch + 2] = x.z;
          v[4 * ch + 3] = x.w;
        }
        tmem_st32(lane_addr + L::kQCol + a * 32, v);
      }
      tmem_st_wait();
      tc_fence_before_sync();
      mbar_arrive(B.q_ready);
      mbar_arrive(B.q_empty);
      return true;
    };
    // Output rows leave through a per-warp staging area so that the global
    // stores are coalesced: each thread holds one head row, but a warp-wide
    // store of one 16-byte piece per row would touch 32 rows at once. A
    // pass stages 64 bytes of each of the warp's 32 rows (16-byte pieces
    // XOR-swizzled by row pair, conflict-free both ways), then every
    // instruction writes 8 rows x 64 contiguous bytes.
    uint8_t* stage = smem + L::kMergeOff + warp * 2048;
    const int st_swz = (lane >> 1) & 3;
    auto stage_put = [&](const uint32_t* a) {
      uint4* r = reinterpret_cast<uint4*>(stage + lane * 64);
#pragma unroll
      for (int v = 0; v < 4; ++v) r[v ^ st_swz] = make_uint4(a[4 * v], a[4 * v + 1], a[4 * v + 2], a[4 * v + 3]);
      __syncwarp();
    };
    // piece k of the coalesced write-out: row 8k + lane/4, 16-byte piece lane%4
    auto stage_get = [&](int k, int& r, int& piece) -> uint4 {
      r = 8 * k + (lane >> 2);
      piece = lane & 3;
      return reinterpret_cast<const uint4*>(stage + r * 64)[piece ^ ((r >> 1) & 3)];
    };
    int c = 0, x = 0, n_o = 0;
    bool ok = copy_q(), final_seen = false;
    float m = -INFINITY, l = 0.f;
    int unit_subs = 0;
    uint32_t s0[32];
    while (ok && !final_seen) {
      const int slot = c & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(B.tab_full + slot, (c >> 1) & 1, abort_flag, P.dev_status, P.wait_ns))) {
        ok = false;
        break;
      }
      const ChunkDesc d = desc[slot];
      mbar_arrive(B.tab_empty + slot);
      ++c;
      final_seen = (d.flags & kFlagFinal) != 0;
      if (d.flags & kFlagFirst) {
        unit_subs = 0;
        // the sink logit seeds the max of every slice (any reference point
        // is exact; this one is usually within the bound of the scores) but
        // joins the denominator only once, in slice 0
        m = sink2;
        l = (d.split == 0 && sink2 > -INFINITY) ? 1.f : 0.f;
      }
      // the chunk's keys in half tiles of kSub, as the UMMA issuer cuts them
      const int ntiles = ceil_tiles(d.nkeys);
      for (int t = 0; ok && t < ntiles; ++t) {
        const int nv_tile = min(kT, d.nkeys - t * kT);
        const int nsub = (nv_tile + kSub - 1) / kSub;
        for (int hf = 0; hf < nsub; ++hf, ++x, ++unit_subs) {
          // tcgen05.ld/st are warp-collective: keep every branch warp-uniform
          if (!__all_sync(0xffffffffu,
                          mbar_wait(B.s_full + (x & 1), (x >> 1) & 1, abort_flag, P.dev_status, P.wait_ns))) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const int nv = min(kSub, nv_tile - hf * kSub);
          const uint32_t s_col = lane_addr + L::kSCol + (x & 1) * kSub;
          // Speculative pass: P with the running max as it stands. Only when
          // some row's sum leaves the bound (NaN and +inf, from a max still
          // at -inf, included) is the exact max taken and P recomputed, so
          // the max reduction stays off the common path. S is still intact
          // in TMEM for that second pass.
          auto load_s = [&]() {
            tmem_ld32(s_col, s0);
            tmem_ld_wait(s0);
            if (nv < kSub) {   // columns past the set: -inf, so they add nothing
#pragma unroll
              for (int cc = 0; cc < 32; ++cc)
                if (cc >= nv) s0[cc] = __float_as_uint(-INFINITY);
            }
          };
          uint32_t pk[16];
          auto exp_pass = [&]() -> float {
            const float neg_m = -m;
            float sum4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int cc = 0; cc < 16; ++cc) {
              const float p0 = exp2_approx(fmaf(__uint_as_float(s0[2 * cc]), P.scale_log2, neg_m));
              const float p1 = exp2_approx(fmaf(__uint_as_float(s0[2 * cc + 1]), P.scale_log2, neg_m));
              sum4[cc & 3] += p0 + p1;
              pk[cc] = pack_bf16x2(p0, p1);
            }
            return (sum4[0] + sum4[1]) + (sum4[2] + sum4[3]);
          };
          load_s();
          float lsum = exp_pass();
          const bool flag = row_ok && !(lsum <= kSpecBound);
          if (__any_sync(0xffffffffu, flag)) {
            load_s();
            // row max: eight independent chains of 3-input max and a tree
            float mx8[8];
#pragma unroll
            for (int k = 0; k < 8; ++k)
              mx8[k] = fmax3(__uint_as_float(s0[k]), __uint_as_float(s0[k + 8]), __uint_as_float(s0[k + 16]));
#pragma unroll
            for (int k = 0; k < 8; ++k) mx8[k] = fmaxf(mx8[k], __uint_as_float(s0[k + 24]));
            const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                                   fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
            const float tmax = mx * P.scale_log2;
            // a flagged row's max lies above its running max
            const bool move = flag && (tmax > m || m == -INFINITY);
            const float alpha = !move ? 1.f : (m == -INFINITY ? 0.f : exp2_approx(m - tmax));
            l *= alpha;
            if (move) m = tmax;
            if (unit_subs > 0 && __any_sync(0xffffffffu, move)) {
              // rows whose max moved rescale their O row (alpha = 1
              // elsewhere), once the PV of the previous half tile has
              // completed: phases before it have, the next one cannot have
              // (it needs this half's P), so the parity names it
              if (!__all_sync(0xffffffffu, mbar_wait(B.o_ready, (x - 1) & 1, abort_flag, P.dev_status,
                                                     P.wait_ns))) {
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
                for (int cc = 0; cc < 32; ++cc) o[cc] = __float_as_uint(__uint_as_float(o[cc]) * alpha);
                tmem_st32(lane_addr + L::kOCol + c0, o);
              }
            }
            lsum = exp_pass();
          }
          l += lsum;
          tmem_st16(s_col, pk);   // P over the first kSub/2 columns of this S buffer
          tmem_st_wait();
          tc_fence_before_sync();
          mbar_arrive(B.p_ready + (x & 1));
        }
      }
      const bool have_o = unit_subs > 0;
      if (!ok || !(d.flags & kFlagLast)) continue;
      // The next unit's Q goes to TMEM first (every QK^T of this unit has
      // completed: its S was seen), so its first QK^T overlaps this epilogue.
      if (!final_seen && !copy_q()) {
        ok = false;
        break;
      }

      // ---- epilogue of the unit
      if (have_o) {
        if (!__all_sync(0xffffffffu, mbar_wait(B.o_done, n_o & 1, abort_flag, P.dev_status, P.wait_ns))) {
          ok = false;
          break;
        }
        ++n_o;
        tc_fence_after_sync();
      }
      const int i = d.i;
      if (S == 1) {
        const float inv_l = l > 0.f ? 1.f / l : 0.f;
        uint16_t* obase = P.out + (static_cast<int64_t>(i) * P.num_heads + head0) * D;
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t o[32];
          if (have_o) {
            tmem_ld32(lane_addr + L::kOCol + c0, o);
            tmem_ld_wait(o);
          } else {
#pragma unroll
            for (int cc = 0; cc < 32; ++cc) o[cc] = 0u;
          }
          uint32_t pk[16];
#pragma unroll
          for (int cc = 0; cc < 16; ++cc)
            pk[cc] = pack_bf16x2(__uint_as_float(o[2 * cc]) * inv_l, __uint_as_float(o[2 * cc + 1]) * inv_l);
          stage_put(pk);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            int r, piece;
            const uint4 v = stage_get(k, r, piece);
            if (warp * 32 + r < heads_here)
              *reinterpret_cast<uint4*>(obase + static_cast<int64_t>(warp * 32 + r) * D + c0 + piece * 8) = v;
          }
          __syncwarp();   // the stage is rewritten by the next pass
        }
        if (row_ok)
          P.lse[static_cast<int64_t>(i) * P.num_heads + h] = l > 0.f ? (m + log2_approx(l)) * kLn2 : -INFINITY;
      } else if (P.cluster_merge) {
        // this CTA's (m, l) rows for the cluster merge at the end; O stays
        // in TMEM
        reinterpret_cast<float2*>(smem + L::kMergeOff)[row] = make_float2(m, l);
        if (tid == 0) *reinterpret_cast<int*>(smem + L::kMiscOff + 12) = have_o ? 1 : 0;
      } else {
        // partial result of this slice (no normalisation); the last slice
        // of the query to finish merges all of them
        const int64_t unit = static_cast<int64_t>(i) * S + d.split;
        float* pbase = P.part_o + (unit * P.num_heads + head0) * D;
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t o[32];
          if (have_o) {
            tmem_ld32(lane_addr + L::kOCol + c0, o);
            tmem_ld_wait(o);
          } else {
#pragma unroll
            for (int cc = 0; cc < 32; ++cc) o[cc] = 0u;
          }
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {   // 16 fp32 columns (64 bytes) per pass
            stage_put(o + 16 * hf);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              int r, piece;
              const uint4 v = stage_get(k, r, piece);
              if (warp * 32 + r < heads_here)
                *reinterpret_cast<uint4*>(pbase + static_cast<int64_t>(warp * 32 + r) * D + c0 + 16 * hf + piece * 4) = v;
            }
            __syncwarp();
          }
        }
        if (row_ok) P.part_ml[unit * P.num_heads + h] = make_float2(m, l);
        __threadfence();
        if (!gsync()) {
          ok = false;
          break;
        }
        if (tid == 0) *ticket_slot = atomicAdd(P.tickets + static_cast<int64_t>(i) * gridDim.y + blockIdx.y, 1u);
        if (!gsync()) {
          ok = false;
          break;
        }
        const bool merge = *ticket_slot == static_cast<uint32_t>(S - 1);
        if (!gsync()) {   // ticket_slot is reused by the next unit
          ok = false;
          break;
        }
        if (merge) {
          // exact merge of the S slices: LSE = M + log2(L), O = sum_s w_s O_s
          // with w_s = 2^(m_s - M) / L. Thread h first turns its head's
          // (m_s, l_s) into the weights (in shared memory), then the 128
          // threads sum the partial rows column-wise with coalesced float4
          // loads, all loads of a batch issued before its stores.
          __threadfence();
          float* wl = reinterpret_cast<float*>(smem + L::kMergeOff);   // [kAttnMaxSplits][128]
          if (row_ok) {
            float M = -INFINITY;
            for (int s = 0; s < S; ++s) {
              const float2 ml = __ldcg(P.part_ml + (static_cast<int64_t>(i) * S + s) * P.num_heads + h);
              if (ml.y > 0.f) M = fmaxf(M, ml.x);
            }
            float Lsum = 0.f;
            for (int s = 0; s < S; ++s) {
              const float2 ml = __ldcg(P.part_ml + (static_cast<int64_t>(i) * S + s) * P.num_heads + h);
              const float w = (ml.y > 0.f) ? exp2_approx(ml.x - M) : 0.f;
              wl[s * 128 + row] = w;
              Lsum += w * ml.y;
            }
            const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
            for (int s = 0; s < S; ++s) wl[s * 128 + row] *= inv;
            P.lse[static_cast<int64_t>(i) * P.num_heads + h] =
                Lsum > 0.f ? (M + log2_approx(Lsum)) * kLn2 : -INFINITY;
          }
          if (!gsync()) {
            ok = false;
            break;
          }
          constexpr int kF4 = D / 4;                   // float4 per row
          constexpr int kRowsPerPass = kSoftThreads / kF4;
          constexpr int kBatch = 4;                    // row passes whose loads are in flight together
          const int rsub = tid / kF4, c4 = tid % kF4;
          const float4* part4 = reinterpret_cast<const float4*>(P.part_o);
#pragma unroll 1
          for (int r0 = 0; r0 < heads_here; r0 += kRowsPerPass * kBatch) {
            float4 acc[kBatch];
#pragma unroll
            for (int q = 0; q < kBatch; ++q) acc[q] = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int s = 0; s < S; ++s) {
#pragma unroll
              for (int q = 0; q < kBatch; ++q) {
                const int hr = r0 + q * kRowsPerPass + rsub;
                if (hr >= heads_here) continue;
                const float w = wl[s * 128 + hr];
                const float4 v = __ldcg(part4 + ((static_cast<int64_t>(i) * S + s) * P.num_heads + head0 + hr) * kF4 + c4);
                acc[q].x = fmaf(w, v.x, acc[q].x);
                acc[q].y = fmaf(w, v.y, acc[q].y);
                acc[q].z = fmaf(w, v.z, acc[q].z);
                acc[q].w = fmaf(w, v.w, acc[q].w);
              }
            }
#pragma unroll
            for (int q = 0; q < kBatch; ++q) {
              const int hr = r0 + q * kRowsPerPass + rsub;
              if (hr >= heads_here) continue;
              *reinterpret_cast<uint2*>(P.out + (static_cast<int64_t>(i) * P.num_heads + head0 + hr) * D + 4 * c4) =
                  make_uint2(pack_bf16x2(acc[q].x, acc[q].y), pack_bf16x2(acc[q].z, acc[q].w));
            }
          }
          if (!gsync()) {   // wl and the staging areas are reused next
            ok = false;
            break;
          }
        }
      }
    }
    cta_finish<D>(P, true, smem, sbase, tmem, tid, warp, S, heads_here, head0);
  }
}

template <int D, bool kFp8>
cudaError_t launch_d(const Params& P, int head_tiles, cudaStream_t stream) {
  using L = Layout<D>;
  static bool configured = false;
  if (!configured) {
    cudaError_t err = cudaFuncSetAttribute(sparse_sink_attn_kernel<D, kFp8>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes);
    if (err != cudaSuccess) return err;
    configured = true;
  }
  const int64_t units = static_cast<int64_t>(P.n_queries) * P.num_splits;
  if (P.cluster_merge) {
    // one unit per CTA, the S slices of a query in one cluster
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(units), head_tiles);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = L::kBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(P.num_splits);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t err = cudaLaunchKernelEx(&cfg, sparse_sink_attn_kernel<D, kFp8>, P);
    if (err != cudaSuccess) return err;
    return cudaGetLastError();
  }
  const int64_t slots = std::max<int64_t>(1, (2 * static_cast<int64_t>(device_sm_count())) / head_tiles);
  dim3 grid(static_cast<unsigned>(std::min<int64_t>(units, slots)), head_tiles);
  sparse_sink_attn_kernel<D, kFp8><<<grid, kThreads, L::kBytes, stream>>>(P);
  return cudaGetLastError();
}

}  // namespace

size_t attn_workspace_bytes(int32_t n_queries, int32_t num_heads, int32_t head_dim,
                            int32_t num_splits) {
  if (num_splits <= kAttnMaxClusterSplits) return 0;   // unsplit, or merged within a cluster
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
  memset(&P, 0, sizeof P);
  if (tensor_map_encoder() == nullptr) return cudaErrorNotSupported;
  P.q_box_rows = std::min(128, a.num_heads);
  const int64_t raw_rows = a.raw_num_pages * a.raw_page_size;
  if (!encode_q(&P.tm_q, a.q, a.n_queries, a.num_heads, a.head_dim, a.q_stride_tok, a.q_stride_head,
                P.q_box_rows) ||
      !encode_pool(&P.tm_k_raw, a.k_raw, raw_rows, a.head_dim) ||
      !encode_pool(&P.tm_v_raw, a.v_raw, raw_rows, a.head_dim))
    return cudaErrorInvalidValue;
  if (a.pt_cmp != nullptr && a.k_cmp_fp8 == nullptr) {
    const int64_t cmp_rows = a.cmp_num_pages * a.cmp_page_size;
    if (!encode_pool(&P.tm_k_cmp, a.k_cmp, cmp_rows, a.head_dim) ||
        !encode_pool(&P.tm_v_cmp, a.v_cmp, cmp_rows, a.head_dim))
      return cudaErrorInvalidValue;
  }
  P.k_raw = reinterpret_cast<const uint8_t*>(a.k_raw);
  P.v_raw = reinterpret_cast<const uint8_t*>(a.v_raw);
  P.k_cmp = a.k_cmp_fp8 == nullptr ? reinterpret_cast<const uint8_t*>(a.k_cmp) : nullptr;
  P.v_cmp = a.k_cmp_fp8 == nullptr ? reinterpret_cast<const uint8_t*>(a.v_cmp) : nullptr;
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
  P.k_cmp8 = a.k_cmp_fp8;
  P.v_cmp8 = a.v_cmp_fp8;
  P.k_cmp_sc = a.k_cmp_scale;
  P.v_cmp_sc = a.v_cmp_scale;
  P.fp8_fnuz = a.fp8_fnuz ? 1 : 0;
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
  P.wait_ns = attn_wait_limit_ns();
  P.stall = attn_stall() ? 1 : 0;
  const int head_tiles = (a.num_heads + 127) / 128;
  P.part_o = nullptr;
  P.part_ml = nullptr;
  P.tickets = nullptr;
  P.cluster_merge = (a.num_splits > 1 && a.num_splits <= kAttnMaxClusterSplits) ? 1 : 0;
  if (a.num_splits > kAttnMaxClusterSplits) {
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
  const bool fp8 = a.k_cmp_fp8 != nullptr;
  if (a.head_dim == 128)
    return fp8 ? launch_d<128, true>(P, head_tiles, stream) : launch_d<128, false>(P, head_tiles, stream);
  return fp8 ? launch_d<64, true>(P, head_tiles, stream) : launch_d<64, false>(P, head_tiles, stream);
}

}  // namespace spa
