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
//   S  = Q[128 x d] . K_tile[64 x d]^T      tcgen05.mma, Q in TMEM, K in SMEM
//   P  = exp2(S*scale*log2e - m)  (BF16)    softmax warps, TMEM -> regs -> TMEM
//   O += P[128 x 64] . V_tile[64 x d]        tcgen05.mma, P in TMEM, V in SMEM
// Both products take their A operand from TMEM: measured on B200, an
// M = 128, N = 64 product with both operands in shared memory is bound by
// shared-memory bandwidth at two thirds of the tensor rate, while with A in
// TMEM it runs at the full rate. The sink seeds the running max and the
// denominator (m = sink*log2e, l = 1), so it is counted exactly once and
// never multiplies a V row.
//
// Persistent CTAs (two per SM) walk their units in a fixed stride; the two
// CTAs of an SM interleave on the tensor core and on the exp unit. Warp
// roles (256 threads):
//   warps 0-3  softmax + epilogue; thread t owns head row t = TMEM lane t.
//              They also move each unit's Q from shared memory into TMEM.
//   warp  4    TMEM allocation; lane 0 issues every UMMA and commit
//   warp  5    resolver: for a chunk of up to 640 keys of a unit it loads
//              the keys, looks their pages up and writes the physical row
//              of every key (bit 31 = raw pool) to a double-buffered table,
//              plus a chunk descriptor that every other role follows. All
//              dependent global loads of the gather happen here, ahead of
//              the copies.
//   warp  6    K gather (and Q): TMA tile::gather4 loads, four rows of one
//              pool per instruction, into a 2-stage ring, 128-byte swizzled
//              by the tensor map into the K-major layout of the UMMA
//              descriptors; rows outside a pool (padding, faulty keys) are
//              zero-filled by the TMA. Q arrives as TMA boxes; the first
//              unit's Q is requested at once (the unit is known from the
//              block index), while the resolver is still fetching keys.
//   warp  7    V gather, into its own 2-stage ring
// (Measured on B200 for the ratio-4 prefill: the same kernel with 16-byte
// cp.async gathers from eight warps per CTA ran 1.24 ms against 1.0 ms
// with TMA gather4 from one warp per operand: the copy warps took issue
// slots and registers the softmax needs.)
// TMEM columns: S/P [0,64), Q [64, 64 + d/2) as packed BF16 pairs, O after.
// S is single-buffered: QK^T of tile g+1 is issued after PV of tile g, and
// the UMMAs of a CTA run in issue order, so P(g) is read before S(g+1)
// overwrites it; the other CTA on the SM fills the tensor core meanwhile.
// The softmax first takes P with the running max as it stands and only
// recomputes a tile whose row sum leaves a fixed bound (see kSpecBound);
// O/l and LSE use the same max, so the result is exact in exact arithmetic.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <type_traits>

#include "attn_common.cuh"

namespace spa {
namespace {

using namespace attn;

constexpr int kStagesK = 2;
constexpr int kStagesV = 2;
constexpr int kSoftThreads = 128;
constexpr int kMmaWarp = 4;
constexpr int kResolverWarp = 5;
constexpr int kKWarp0 = 6;                       // K (and Q) producer
constexpr int kVWarp0 = 7;                       // V producer
constexpr int kThreads = 256;
constexpr uint32_t kTmemCols = 256;
// A tile whose row sum of P, taken with the running max as it stands,
// exceeds 2^16 (or is not a number) is recomputed with its exact max. P
// therefore stays below 2^16: harmless in BF16 and in the FP32 sums, whose
// relative precision does not depend on magnitude.
constexpr float kSpecBound = 65536.0f;
// consumers of a chunk descriptor: K warp, V warp, MMA thread, softmax
constexpr uint32_t kTabConsumers = 32 + 32 + 1 + kSoftThreads;

struct Params {
  // TMA descriptors (passed as a __grid_constant__ parameter)
  CUtensorMap tm_q;       // 3D {d, H, N}, box {64, q_box_rows, 1}
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
  // s_full, p_ready, o_done, mma_done, soft_sync[2]
  static constexpr int kNumBars = 2 + 2 + 3 + 2 * kStagesK + 2 * kStagesV + 1 + 1 + 1 + 1 + 2;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  // misc: TMEM slot, abort flag, ticket, have_o, the testing stall barrier
  // at +16 and the cluster merge's receive barrier at +24
  static constexpr int kUsed = kMiscOff + 32;
  // + alignment slack; at least 80 KB so that no more than two CTAs share an
  // SM (TMEM holds two 256-column allocations)
  static constexpr int kBytes = (kUsed + 1024) < 80 * 1024 ? 80 * 1024 : (kUsed + 1024);
  static constexpr uint32_t kSCol = 0;
  static constexpr uint32_t kQCol = kT;
  static constexpr uint32_t kOCol = kT + D / 2;
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
  uint64_t* s_full;     // S of the current tile (also: every earlier UMMA done)
  uint64_t* p_ready;    // P of the current tile in TMEM
  uint64_t* o_done;     // last PV of a unit complete
  uint64_t* mma_done;
  // [2]: barrier of the softmax threads, the two used in turn. An mbarrier
  // rather than a named barrier so that the wait is bounded: a thread that
  // gave up elsewhere cannot leave the others stuck.
  uint64_t* soft_sync;
};

template <int D, bool kFp8>
__global__ void __launch_bounds__(kThreads, 2) sparse_sink_attn_kernel(const __grid_constant__ Params P) {
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
  B.p_ready = B.s_full + 1;
  B.o_done = B.p_ready + 1;
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
      mbar_init(B.tab_full + s, 32);
      mbar_init(B.tab_empty + s, kTabConsumers);
      mbar_init(B.soft_sync + s, kSoftThreads);
    }
    mbar_init(B.q_full, 1);
    mbar_init(B.q_empty, kSoftThreads);
    mbar_init(B.q_ready, kSoftThreads);
    for (int s = 0; s < kStagesK; ++s) {
      mbar_init(B.k_full + s, 1);
      mbar_init(B.k_empty + s, 1);
    }
    for (int s = 0; s < kStagesV; ++s) {
      mbar_init(B.v_full + s, 1);
      mbar_init(B.v_empty + s, 1);
    }
    mbar_init(B.s_full, 1);
    mbar_init(B.p_ready, kSoftThreads);
    mbar_init(B.o_done, 1);
    mbar_init(B.mma_done, 1);
    *abort_flag = 0;
    mbar_init(reinterpret_cast<uint64_t*>(smem + L::kMiscOff + 16), 1);   // never arrived at
    mbar_init(reinterpret_cast<uint64_t*>(smem + L::kMiscOff + 24), 1);   // cluster merge: rows received
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
  // everything above is private to the CTA; every global read below may
  // depend on the previous kernel of the stream (the sets, the pools, Q)
  grid_dep_wait();

  if (warp == kResolverWarp) {
    // ================================================= resolver
    // testing stall: a wait that only its limit ends, then the CTA unwinds
    if (P.stall) mbar_wait(reinterpret_cast<uint64_t*>(smem + L::kMiscOff + 16), 0, abort_flag, P.dev_status, P.wait_ns);
    resolver_loop(P, S, tab, desc, B.tab_full, B.tab_empty, abort_flag, lane);
  } else if (warp == kKWarp0 || warp == kVWarp0) {
    // ================================================= K / V gather (TMA)
    // A tile is 16 four-row groups x D/64 column halves = "jobs"; lane j
    // issues one TMA tile::gather4 for job j (four rows of one pool, 512
    // bytes). A group whose four keys come from both pools (at most one per
    // unit: compressed groups precede window tokens) is loaded row by row.
    // Rows past the chunk's keys and rows of faulty keys are outside the
    // tensor and zero-filled. Lane 0 of the K warp also loads each unit's Q
    // (every unit, empty ones included, so that the Q phases of all roles
    // stay in step).
    const bool is_k = warp == kKWarp0;
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
    bool final_seen = false, first_q_issued = false;
    if (is_k) {
      // The CTA's first unit is unit blockIdx.x (units are strided over the
      // CTAs): its Q is loaded at once, while the resolver fetches its keys.
      if (lane == 0) {
        mbar_arrive_expect_tx(B.q_full, P.q_box_rows * 128 * kHalves);
        for (int hb = 0; hb < kHalves; ++hb)
          tma_load_3d(sbase + L::kQOff + hb * (128 * 128), &P.tm_q, B.q_full, hb * 64, head0,
                      static_cast<int32_t>(blockIdx.x / S));
      }
      first_q_issued = true;
      qc = 1;
    }
    while (!final_seen) {
      const int slot = c & 1;
      if (!mbar_wait(B.tab_full + slot, (c >> 1) & 1, abort_flag, P.dev_status, P.wait_ns)) break;
      const ChunkDesc d = desc[slot];
      final_seen = (d.flags & kFlagFinal) != 0;
      const uint32_t* t_rows = tab + slot * kChunkKeys;
      const int ntiles = ceil_tiles(d.nkeys);
      bool ok = true;
      if (is_k && (d.flags & kFlagFirst) && first_q_issued) {
        first_q_issued = false;   // the first unit's Q is on its way
      } else if (is_k && (d.flags & kFlagFirst)) {
        // the landing area is free once the previous Q has moved to TMEM
        ok = mbar_wait(B.q_empty, (qc & 1) ^ 1, abort_flag, P.dev_status, P.wait_ns);
        if (ok && lane == 0) {
          mbar_arrive_expect_tx(B.q_full, P.q_box_rows * 128 * kHalves);
          for (int hb = 0; hb < kHalves; ++hb)
            tma_load_3d(sbase + L::kQOff + hb * (128 * 128), &P.tm_q, B.q_full, hb * 64, head0, d.i);
        }
        if (ok) ++qc;
      }
      if constexpr (!kFp8) {
        for (int t = 0; ok && t < ntiles; ++t, ++g) {
          const int stage = g % nst;
          if (!mbar_wait(empty + stage, ((g / nst) & 1) ^ 1, abort_flag, P.dev_status, P.wait_ns)) { ok = false; break; }
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
            for (int k = 0; k < 4; ++k)   // rows outside the tensor are zero-filled
              y[k] = e[k] == kInvalidRow ? -1 : static_cast<int32_t>(e[k] & ~kRawBit);
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
      } else {
        // Fused FP8 decode. Raw (window) rows and zero rows (past the set,
        // faulty keys) still come by TMA; compressed rows are read as E4M3
        // codes and scales with plain loads (all of a tile's loads in flight
        // together), decoded exactly as the page decode does, and written
        // into the same 128-byte swizzled BF16 layout. The tile is complete
        // once the TMA bytes have landed and lane 0 has arrived after every
        // lane's shared-memory writes. (Staging the codes through cp.async
        // in the destination stage, and issuing the next tile's loads before
        // this tile's decode, both measured slower on B200.)
        constexpr int kPieces = D / 16;   // 16 codes per piece
        constexpr int kPerLane = kT * kPieces / 32;
        static_assert(kPieces * 16 == D && (D == 64 || D == 128), "16 codes per piece, one or two halves");
        const uint8_t* pool8 = is_k ? P.k_cmp8 : P.v_cmp8;
        const float* psc = is_k ? P.k_cmp_sc : P.v_cmp_sc;
        // Lane l always handles piece l % kPieces (16 codes) of rows
        // (l + 32 j) / kPieces.
        const int piece = lane % kPieces;
        for (int t = 0; ok && t < ntiles; ++t, ++g) {
          const int stage = g % nst;
          if (!mbar_wait(empty + stage, ((g / nst) & 1) ^ 1, abort_flag, P.dev_status, P.wait_ns)) { ok = false; break; }
          const int nv = min(kT, d.nkeys - t * kT);
          const uint32_t* trow = t_rows + t * kT;
          uint32_t tx = 0;
          uint32_t e[4];
          bool fp8_row[4] = {false, false, false, false};
          if (issuer) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const int r = 4 * grp + k;
              e[k] = r < nv ? trow[r] : kInvalidRow;
              fp8_row[k] = e[k] != kInvalidRow && !(e[k] & kRawBit);
              if (!fp8_row[k]) tx += 128;
            }
          }
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) tx += __shfl_xor_sync(0xffffffffu, tx, off);
          if (lane == 0) mbar_expect_tx(full + stage, tx);
          __syncwarp();
          if (issuer) {
            int32_t y[4];
#pragma unroll
            for (int k = 0; k < 4; ++k)
              y[k] = (e[k] == kInvalidRow || fp8_row[k]) ? -1 : static_cast<int32_t>(e[k] & ~kRawBit);
            const uint32_t dst = ring + stage * L::kTileBytes + half * (kT * 128) + (4 * grp) * 128;
            if (!(fp8_row[0] || fp8_row[1] || fp8_row[2] || fp8_row[3])) {
              tma_gather4(dst, map_raw, full + stage, half * 64, y[0], y[1], y[2], y[3]);
            } else {
#pragma unroll
              for (int k = 0; k < 4; ++k)
                if (!fp8_row[k]) tma_load_2d(dst + k * 128, map_raw, full + stage, half * 64, y[k]);
            }
          }
          uint8_t* tile = smem + (is_k ? L::kKOff : L::kVOff) + stage * L::kTileBytes;
          // Every load first (one round trip), then the codes and scales are
          // staged in the FP8 rows' own bytes of the destination tile
          // (d = 128: the codes over the row's second half, the scales at the
          // start of its first half; d = 64: the codes in the row's last 64
          // bytes, the scale in its first 4), bytes no TMA row and no other
          // row touches, and a rolled loop decodes 32 / kPieces rows per
          // step, reading a step's staged bytes before any lane overwrites
          // them. The rolled loop keeps the decode's code small: unrolled,
          // it was fetched anew for every tile and took most of the tile's
          // time.
          auto code_off = [](int r, int pc) { return (D == 128 ? kT * 128 : 64) + r * 128 + pc * 16; };
          uint4 raw[kPerLane];
          float sc[kPerLane];
#pragma unroll
          for (int j = 0; j < kPerLane; ++j) {   // every load first
            const int r = (lane + 32 * j) / kPieces;
            const uint32_t er = r < nv ? trow[r] : kInvalidRow;
            raw[j] = make_uint4(0u, 0u, 0u, 0u);
            sc[j] = 0.f;
            if (er != kInvalidRow && !(er & kRawBit)) {
              const int64_t row8 = er;
              raw[j] = __ldg(reinterpret_cast<const uint4*>(pool8 + row8 * D + piece * 16));
              sc[j] = __ldg(psc + row8 * (D / 64) + (piece * 16) / 64);
            }
          }
#pragma unroll
          for (int j = 0; j < kPerLane; ++j) {
            const int r = (lane + 32 * j) / kPieces;
            const uint32_t er = r < nv ? trow[r] : kInvalidRow;
            if (er == kInvalidRow || (er & kRawBit)) continue;
            *reinterpret_cast<uint4*>(tile + code_off(r, piece)) = raw[j];
            if (piece % 4 == 0) *reinterpret_cast<float*>(tile + r * 128 + (piece / 4) * 4) = sc[j];
          }
          __syncwarp();
          auto decode_all = [&](auto fnuz) {
#pragma unroll 1
            for (int j = 0; j < kPerLane; ++j) {
              const int r = (lane + 32 * j) / kPieces;
              const uint32_t er = r < nv ? trow[r] : kInvalidRow;
              const bool mine = er != kInvalidRow && !(er & kRawBit);
              uint4 code = make_uint4(0u, 0u, 0u, 0u);
              float scale = 0.f;
              if (mine) {
                code = *reinterpret_cast<const uint4*>(tile + code_off(r, piece));
                scale = *reinterpret_cast<const float*>(tile + r * 128 + (piece / 4) * 4);
              }
              __syncwarp();   // this step's rows are read before any lane writes them
              if (mine) {
                uint32_t o[8];
                decode_e4m3x16<decltype(fnuz)::value>(code, scale, o);
                const int hf = (piece * 16) / 64, ch0 = ((piece * 16) % 64) / 8;
                uint8_t* row_ptr = tile + hf * (kT * 128) + r * 128;
                *reinterpret_cast<uint4*>(row_ptr + ((ch0 ^ (r & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
                *reinterpret_cast<uint4*>(row_ptr + (((ch0 + 1) ^ (r & 7)) << 4)) = make_uint4(o[4], o[5], o[6], o[7]);
              }
            }
          };
          if (P.fp8_fnuz) decode_all(std::true_type{});
          else decode_all(std::false_type{});
          fence_proxy_async_smem();   // generic-proxy writes -> the UMMA's reads
          __syncwarp();
          if (lane == 0) mbar_arrive(full + stage);
        }
      }
      mbar_arrive(B.tab_empty + slot);
      ++c;
      if (!ok) break;
    }
    // every copy this warp started has landed before the CTA can leave (they
    // land even when the roles gave up early; these waits keep the fixed
    // limit): the last two ring stages, and the last Q
    for (int k = 1; k <= nst && k <= g; ++k)
      mbar_wait(full + (g - k) % nst, ((g - k) / nst) & 1, nullptr, P.dev_status);
    if (is_k && qc > 0) mbar_wait(B.q_full, (qc - 1) & 1, nullptr, P.dev_status);
  } else if (warp == kMmaWarp) {
    // ================================================= UMMA issuer
    // Per tile: S = Q K^T (A = Q from TMEM), then, once P is in TMEM,
    // O += P V (A = P from TMEM). s_full is committed after the QK^T of a
    // tile, so its arrival also means every earlier UMMA (the previous PV)
    // has completed.
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, kT, 0);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, D, 1);
      int c = 0, g = 0, u = 0;
      bool ok = true, final_seen = false;
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
        for (int t = 0; t < ntiles; ++t, ++g) {
          const int stage = g % kStagesK, st = g % kStagesV;
          if (!mbar_wait(B.k_full + stage, (g / kStagesK) & 1, abort_flag, P.dev_status, P.wait_ns)) { ok = false; break; }
          tc_fence_after_sync();
          const uint32_t k_addr = sbase + L::kKOff + stage * L::kTileBytes;
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint64_t bdesc = smem_desc_sw128(k_addr + (k >> 2) * (kT * 128) + (k & 3) * 32, 16, 1024);
            umma_ts(tmem + L::kSCol, tmem + L::kQCol + k * 8, bdesc, idesc_s, k > 0 ? 1u : 0u);
          }
          tc_commit(B.k_empty + stage);
          tc_commit(B.s_full);
          if (!mbar_wait(B.p_ready, g & 1, abort_flag, P.dev_status, P.wait_ns)) { ok = false; break; }
          if (!mbar_wait(B.v_full + st, (g / kStagesV) & 1, abort_flag, P.dev_status, P.wait_ns)) { ok = false; break; }
          tc_fence_after_sync();
          const uint32_t v_addr = sbase + L::kVOff + st * L::kTileBytes;
          const bool first = (d.flags & kFlagFirst) && t == 0;
#pragma unroll
          for (int k = 0; k < kT / 16; ++k) {
            const uint64_t bdesc = smem_desc_sw128(v_addr + k * 16 * 128, kT * 128, 1024);
            umma_ts(tmem + L::kOCol, tmem + L::kSCol + k * 8, bdesc, idesc_o, (!first || k > 0) ? 1u : 0u);
          }
          tc_commit(B.v_empty + st);
          if ((d.flags & kFlagLast) && t == ntiles - 1) tc_commit(B.o_done);
        }
      }
      // every UMMA has completed before TMEM is released
      tc_commit(B.mma_done);
      mbar_wait(B.mma_done, 0, nullptr, P.dev_status);
    }
  } else {
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
    int c = 0, g = 0, n_o = 0;
    bool ok = copy_q(), final_seen = false;
    float m = -INFINITY, l = 0.f;
    int unit_tiles = 0;
    uint32_t s0[32], s1[32];
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
        unit_tiles = 0;
        // the sink logit seeds the max of every slice (any reference point
        // is exact; this one is usually within the bound of the scores) but
        // joins the denominator only once, in slice 0
        m = sink2;
        l = (d.split == 0 && sink2 > -INFINITY) ? 1.f : 0.f;
      }
      const int ntiles = ceil_tiles(d.nkeys);
      for (int t = 0; t < ntiles; ++t, ++g, ++unit_tiles) {
        // tcgen05.ld/st are warp-collective: keep every branch warp-uniform
        if (!__all_sync(0xffffffffu, mbar_wait(B.s_full, g & 1, abort_flag, P.dev_status, P.wait_ns))) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const int nv = min(kT, d.nkeys - t * kT);
        // Speculative pass: P with the running max as it stands. Only when
        // some row's tile sum leaves the bound (NaN and +inf, from a max
        // still at -inf, included) is the exact tile max taken and P
        // recomputed, so the max reduction stays off the common path. S is
        // still intact in TMEM for that second pass.
        auto load_s = [&]() {
          tmem_ld32(lane_addr + L::kSCol, s0);
          tmem_ld32(lane_addr + L::kSCol + 32, s1);
          tmem_ld_wait(s0);
          tmem_ld_wait(s1);
          if (nv < kT) {   // columns past the set: -inf, so they add nothing
#pragma unroll
            for (int cc = 0; cc < 32; ++cc) {
              if (cc >= nv) s0[cc] = __float_as_uint(-INFINITY);
              if (cc + 32 >= nv) s1[cc] = __float_as_uint(-INFINITY);
            }
          }
        };
        uint32_t pk[32];
        auto exp_pass = [&]() -> float {
          const float neg_m = -m;
          float sum4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int cc = 0; cc < 16; ++cc) {
            const float p0 = exp2_approx(fmaf(__uint_as_float(s0[2 * cc]), P.scale_log2, neg_m));
            const float p1 = exp2_approx(fmaf(__uint_as_float(s0[2 * cc + 1]), P.scale_log2, neg_m));
            const float p2 = exp2_approx(fmaf(__uint_as_float(s1[2 * cc]), P.scale_log2, neg_m));
            const float p3 = exp2_approx(fmaf(__uint_as_float(s1[2 * cc + 1]), P.scale_log2, neg_m));
            sum4[cc & 3] += (p0 + p1) + (p2 + p3);
            pk[cc] = pack_bf16x2(p0, p1);
            pk[cc + 16] = pack_bf16x2(p2, p3);
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
            mx8[k] = fmax3(__uint_as_float(s0[k]), __uint_as_float(s1[k]), __uint_as_float(s0[k + 8]));
#pragma unroll
          for (int k = 0; k < 8; ++k)
            mx8[k] = fmax3(mx8[k], __uint_as_float(s1[k + 8]), __uint_as_float(s0[k + 16]));
#pragma unroll
          for (int k = 0; k < 8; ++k)
            mx8[k] = fmax3(mx8[k], __uint_as_float(s1[k + 16]), __uint_as_float(s0[k + 24]));
#pragma unroll
          for (int k = 0; k < 8; ++k) mx8[k] = fmaxf(mx8[k], __uint_as_float(s1[k + 24]));
          const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                                 fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
          const float tmax = mx * P.scale_log2;
          // a flagged row's tile max lies above its running max
          const bool move = flag && (tmax > m || m == -INFINITY);
          const float alpha = !move ? 1.f : (m == -INFINITY ? 0.f : exp2_approx(m - tmax));
          l *= alpha;
          if (move) m = tmax;
          if (unit_tiles > 0 && __any_sync(0xffffffffu, move)) {
            // rows whose max moved rescale their O row (alpha = 1
            // elsewhere); the previous PV has completed (s_full)
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
        tmem_st32(lane_addr + L::kSCol, pk);   // P overwrites the first 32 columns of S
        tmem_st_wait();
        tc_fence_before_sync();
        mbar_arrive(B.p_ready);
      }
      if (!ok || !(d.flags & kFlagLast)) continue;
      // The next unit's Q goes to TMEM first (every QK^T of this unit has
      // completed: its S was seen), so its first QK^T overlaps this epilogue.
      if (!final_seen && !copy_q()) {
        ok = false;
        break;
      }

      // ---- epilogue of the unit
      const bool have_o = unit_tiles > 0;
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
        // this CTA's (m, l) rows for the cluster merge at the end, into slot
        // `split` of every CTA of the cluster (posted stores, so that after
        // the first cluster barrier every (m, l) is local); O stays in TMEM
        const uint32_t ml_slot = sbase + L::kMergeOff + static_cast<uint32_t>((d.split * 128 + row) * 8);
#pragma unroll 1
        for (int s = 0; s < S; ++s) st_dsmem_f2(dsmem_addr(ml_slot, s), make_float2(m, l));
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
  }

  // ---- teardown: every TMEM access above has completed
  __syncwarp();
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if (P.cluster_merge) {
    // Exact merge of the S slices of query i, CTA `rank` holding slice
    // `rank`: LSE = M + log2(L), O = sum_s w_s O_s with w_s = 2^(m_s - M)/L
    // (page "[WS2] Add CP-aware Attention contract and dispatch metadata",
    // Summary: the deterministic (out, lse) merge). CTA r owns rows
    // [r*per, (r+1)*per) of the output. After the cluster barrier every CTA
    // has all slices' (m, l) of its rows (each slice stored its own into
    // every CTA before the barrier), scales its O rows by its weight and
    // writes each as FP16: its own rows into its receive slot, the others
    // into a staging block per owner, laid out as that owner's slot; one
    // thread then sends each block with one bulk copy into the owner's idle
    // K/V ring (slot = the sender's rank), completing the owner's receive
    // barrier, armed before the cluster barrier for the rows of all other
    // slices. Each owner waits on its barrier, sums its slots in FP32 and
    // writes BF16 O; a sender leaves only once its copies have read their
    // rows. (Posted remote stores from every thread, about 12 bytes per
    // clock per SM on B200, and a second cluster barrier took 3.8 us of a
    // 25 us decode launch.) A weighted row is at most max|v| in magnitude and
    // FP16 keeps 11 bits, more than the BF16 output, at half the bytes of
    // FP32 rows. Every thread of every CTA reaches the cluster barrier: every
    // earlier wait in the kernel is bounded.
    const int rank = static_cast<int>(cluster_ctarank());
    const int i = static_cast<int>(blockIdx.x / S);
    const float2* ml_all = reinterpret_cast<const float2*>(smem + L::kMergeOff);   // [S][128] (m, l)
    static_assert(kAttnMaxClusterSplits * 128 * 8 <= kAttnMaxSplits * 128 * 4, "(m, l) slots fit the merge area");
    const uint32_t rx_addr = sbase + L::kKOff;               // [S][per][D] FP16, 16-byte chunks swizzled by row
    constexpr int kChunks = D / 8;                           // 16-byte chunks per row
    const int per = (128 + S - 1) / S;
    // the slots (S * per <= 128 + S - 1 rows of D FP16) fit the idle K/V rings
    static_assert(L::kTabOff - L::kKOff >= (128 + kAttnMaxClusterSplits - 1) * D * 2,
                  "receive slots fit the idle rings");
    static_assert(L::kTabOff == L::kVOff + kStagesV * L::kTileBytes && L::kVOff == L::kKOff + kStagesK * L::kTileBytes,
                  "rings and tables are contiguous");
    // the rows of this CTA's own slot come by local stores, the others by
    // one bulk copy per sender, staged in the sender's idle rings after the
    // receive slots
    uint64_t* rx_bar = reinterpret_cast<uint64_t*>(smem + L::kMiscOff + 24);
    const int my_rows = min(per, 128 - rank * per);
    if (tid == 0) mbar_arrive_expect_tx(rx_bar, static_cast<uint32_t>((S - 1) * my_rows * D * 2));
    constexpr int kRxMaxBytes = (128 + kAttnMaxClusterSplits - 1) * D * 2;
    const uint32_t stage_addr = rx_addr + kRxMaxBytes;       // [S][per][D] FP16, as the receive slots
    static_assert(2 * kRxMaxBytes <= L::kDescOff - L::kKOff, "receive slots and send staging fit the idle rings");
    __syncwarp();
    cluster_sync_all();                                      // every slice's (m, l) is in place; rings idle
    if (tid < kSoftThreads) {
      const int row = tid;
      float2 ml[kAttnMaxClusterSplits];
#pragma unroll
      for (int s = 0; s < kAttnMaxClusterSplits; ++s)
        ml[s] = s < S ? ml_all[s * 128 + row] : make_float2(-INFINITY, 0.f);
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
      const bool local = owner == rank;
      // own rows: straight into this CTA's slot; the others: into the
      // staging block of their owner, laid out as the owner's slot
      const uint32_t slot = local ? rx_addr + static_cast<uint32_t>(((rank * per + rr) * D) * 2)
                                  : stage_addr + static_cast<uint32_t>(((owner * per + rr) * D) * 2);
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
        for (int v = 0; v < 4; ++v) {   // 8 columns per 16-byte chunk
          const int chunk = (c0 >> 3) + v;
          const int phys = chunk ^ (rr & (kChunks - 1));
          uint32_t h[4];
#pragma unroll
          for (int k = 0; k < 4; ++k)
            h[k] = pack_f16x2(__uint_as_float(o[8 * v + 2 * k]) * scale_own,
                              __uint_as_float(o[8 * v + 2 * k + 1]) * scale_own);
          *reinterpret_cast<uint4*>(smem + (slot - sbase) + phys * 16) = make_uint4(h[0], h[1], h[2], h[3]);
        }
      }
    }
    fence_proxy_async_smem();   // the staged rows (generic writes) -> the bulk copies' reads
    __syncthreads();
    if (tid == 0) {
      for (int o = 0; o < S; ++o) {
        if (o == rank) continue;
        const int rows = min(per, 128 - o * per);
        bulk_copy_to_cluster(dsmem_addr(rx_addr + static_cast<uint32_t>((rank * per * D) * 2), o),
                             stage_addr + static_cast<uint32_t>((o * per * D) * 2),
                             static_cast<uint32_t>(rows * D * 2), dsmem_addr(smem_u32(rx_bar), o));
      }
      bulk_commit_group();
    }
    // every other slice's rows for this CTA have landed (a wait that gives
    // up leaves the status word set and the rows unwritten)
    const bool rx_ok = tid >= kSoftThreads || mbar_wait(rx_bar, 0, abort_flag, P.dev_status, P.wait_ns);
    if (tid < kSoftThreads && rx_ok) {
      const int r0 = min(rank * per, heads_here), r1 = min(r0 + per, heads_here);
      const uint8_t* rx = smem + L::kKOff;
      uint16_t* obase = P.out + (static_cast<int64_t>(i) * P.num_heads + head0) * D;
      const int n_items = (r1 - r0) * kChunks;
      for (int idx = tid; idx < n_items; idx += kSoftThreads) {
        const int rr = idx / kChunks, c = idx % kChunks;
        const int phys = c ^ (rr & (kChunks - 1));
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int s = 0; s < S; ++s) {
          const uint4 v = *reinterpret_cast<const uint4*>(rx + ((s * per + rr) * D) * 2 + phys * 16);
          const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float2 f = unpack_f16x2(w4[k]);
            acc[2 * k] += f.x;
            acc[2 * k + 1] += f.y;
          }
        }
        *reinterpret_cast<uint4*>(obase + static_cast<int64_t>(r0 + rr) * D + 8 * c) =
            make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]), pack_bf16x2(acc[4], acc[5]),
                       pack_bf16x2(acc[6], acc[7]));
      }
    }
  }
  if (P.cluster_merge && tid == 0) bulk_wait_read_all();   // the outgoing copies have read their rows
  if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
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
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(P.num_splits);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // may start early
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    cudaError_t err = cudaLaunchKernelEx(&cfg, sparse_sink_attn_kernel<D, kFp8>, P);
    if (err != cudaSuccess) return err;
    return cudaGetLastError();
  }
  const int64_t slots = std::max<int64_t>(1, (2 * static_cast<int64_t>(device_sm_count())) / head_tiles);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(std::min<int64_t>(units, slots)), head_tiles);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = L::kBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // may start early
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t err = cudaLaunchKernelEx(&cfg, sparse_sink_attn_kernel<D, kFp8>, P);
  if (err != cudaSuccess) return err;
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
