/*
 * spa.h -- C ABI of libspa.so: sparse paged attention with an attention
 * sink, for NVIDIA B200 (sm_100a). The path: the per-token key sets (1), the
 * FP8 page decode (2), the attention forward (3, 3b with the FP8 decode in
 * its gather); around it: the backward (3c), the paged write of new window
 * tokens (4) and the decode of packed 512-wide rows (5).
 *
 * The method (page "Roadmap item 24 - joint compressed/window attention with
 * sink", RL-Kernel PR #628, section "Reuse and arithmetic"): for each query
 * token a KV set is gathered through a page table -- the complete recent
 * window of raw tokens plus compressed-KV entries -- and all heads share it.
 * Compressed KV, window and a per-head sink logit share one softmax
 * denominator; the sink has no V. O is BF16 and LSE is the FP32 natural log
 * of the denominator.
 *
 * Conventions shared by every call
 *  - Pointers are DEVICE pointers unless a comment says otherwise. The
 *    caller owns every buffer; the library never allocates, frees or
 *    synchronises, and never reads device data on the host, so every call
 *    can be captured in a CUDA graph. Work is enqueued on `stream`
 *    (NULL = the legacy default stream).
 *  - BF16 tensors are passed as `uint16_t*` holding the bit patterns.
 *  - Host-side validation is synchronous: a call that returns anything but
 *    SPA_OK has enqueued nothing. `spa_last_error_detail()` names the
 *    failing clause.
 *  - Faults that only the device can see (a page id outside the pool, a
 *    logical index past the page table, a malformed key, an overflow of the
 *    output capacity, a wait that ran out of time) never trap: the kernel
 *    skips the offending entry and ORs a SPA_DEV_* bit into `*dev_status`
 *    (may be NULL, then the bit is dropped). After any fault the call's
 *    outputs are undefined ("poisoned"); do not reuse them.
 *  - Workspaces are caller-provided device memory of at least the size the
 *    matching *_workspace_size() returns; their contents need not be
 *    initialised and are clobbered. One workspace must not be shared by
 *    calls that may run at the same time.
 */
#ifndef SPA_H_
#define SPA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;                     /* == cudaStream_t */
typedef struct CUstream_st* spa_stream_t;

#define SPA_ABI_VERSION 1

typedef enum {
    SPA_OK = 0,
    SPA_ERR_INVALID_ARG = 1,   /* null pointer, negative size, bad ratio/window ...   */
    SPA_ERR_UNSUPPORTED = 2,   /* valid, but not a shape/format this build handles    */
    SPA_ERR_CAPACITY = 3,      /* an output buffer is smaller than the bound          */
    SPA_ERR_WORKSPACE = 4,     /* workspace missing or smaller than required          */
    SPA_ERR_ALIGNMENT = 5,     /* a pointer or stride breaks the 16-byte rule         */
    SPA_ERR_CUDA = 6,          /* a CUDA runtime call failed (e.g. launch)            */
} spa_status;

/* Bits of the device status word. */
#define SPA_DEV_BAD_PAGE  1u   /* page id outside [0, num_pages)                      */
#define SPA_DEV_BAD_INDEX 2u   /* key/position/request outside its table              */
#define SPA_DEV_CAPACITY  4u   /* the key sets overflowed `capacity`                  */
#define SPA_DEV_TIMEOUT   8u   /* a bounded wait inside a kernel ran out              */
#define SPA_DEV_SCRATCH_RACE 16u /* two set builds that may run at the same time used
                                  the same scan scratch (one workspace for both, or
                                  overlapping spa_build_kv_sets_noalloc calls); the
                                  sets of that call are wrong                          */

/* A key is a compressed-group index g (0 <= g < 2^30) or
 * SPA_WINDOW_TAG | t for raw token t (0 <= t < 2^30). Ascending key order is
 * the canonical order of a set: compressed groups first, then the window. */
#define SPA_WINDOW_TAG (1 << 30)

int spa_abi_version(void);
const char* spa_status_string(int status);
/* Host-thread-local text naming the clause that made the last call on this
 * thread fail ("" after a success). */
const char* spa_last_error_detail(void);

/* ------------------------------------------------------------------------
 * 1. spa_build_kv_sets -- per-token KV sets as CSR, canonical order.
 *
 * Defined by "Roadmap item 24", section "Contracts and lifetime" (logical
 * request/position/kind keys, complete windows, C4/C128 group boundaries,
 * canonical KV ordering), and "test: add block-level DeepSeek-V4 attention
 * test" (ROCm/ATOM PR #1723), opening section (layer types: compress ratio
 * 0 = dense, 4 = CSA, 128 = HCA) and "Validation" (top-k truncates only once
 * the complete groups outnumber it).
 *
 * For query i at position p = pos[i]:
 *   window  = { SPA_WINDOW_TAG | t : max(0, p-W+1) <= t <= p }
 *   groups  = none                                  (ratio 0)
 *           = { g : 0 <= g < floor((p+1)/ratio) }   (topk == NULL)
 *           = { topk[i][j] : 0 <= topk[i][j] < floor((p+1)/ratio) } (else),
 *             repeats removed (a group is complete once all `ratio` of its
 *             tokens are at or before p)
 *   set_i   = ascending(groups U window)
 *   indptr[0] = 0, indptr[i+1] = indptr[i] + |set_i|,
 *   indices[indptr[i] .. indptr[i+1]) = set_i.
 *
 * pos      int32 [n_queries], 0 <= pos < 2^30 (else SPA_DEV_BAD_INDEX and an
 *          empty set for that query)
 * window   W >= 1
 * ratio    0, 4 or 128
 * topk     int32 [n_queries, topk_width] row-major, or NULL; entries < 0
 *          are padding. topk_width <= 2048.
 * indptr   int32 [n_queries + 1] (output)
 * indices  int32 [capacity] (output); capacity >= spa_kv_sets_capacity(..)
 *          of the true maximum position is enough. Keys past `capacity`
 *          are dropped and SPA_DEV_CAPACITY is set.
 * workspace >= spa_build_kv_sets_workspace_size(n_queries) bytes.
 * ---------------------------------------------------------------------- */
int64_t spa_kv_sets_capacity(int32_t n_queries, int32_t window, int32_t ratio,
                             int32_t topk_width, int32_t has_topk, int32_t max_pos);
size_t spa_build_kv_sets_workspace_size(int32_t n_queries);
int spa_build_kv_sets(const int32_t* pos, int32_t n_queries, int32_t window, int32_t ratio,
                      const int32_t* topk, int32_t topk_width, int32_t* indptr,
                      int32_t* indices, int64_t capacity, void* workspace,
                      size_t workspace_bytes, uint32_t* dev_status, spa_stream_t stream);

/* ------------------------------------------------------------------------
 * 1b. spa_build_kv_sets_noalloc -- spa_build_kv_sets with no workspace.
 *
 * The pages have no counterpart to this call; it exists for callers that
 * cannot allocate device memory at the point where the sets are built: code
 * that runs inside a host framework which reserves all device memory up
 * front and hands out no scratch (a serving engine's fixed arena, a plugin
 * interface without a workspace argument), or code called while a CUDA
 * graph is being captured, where a fresh allocation would either fail or be
 * baked into the graph.
 *
 * Same arguments, results and device-status bits as spa_build_kv_sets,
 * minus `workspace` / `workspace_bytes`. The scan scratch is a fixed array
 * of 1 MiB + 16 bytes inside the library (every GPU that loads the library
 * keeps it until the process exits), so n_queries is limited to
 * 1,048,576; larger calls return SPA_ERR_UNSUPPORTED without enqueueing
 * anything. The call allocates nothing (no cudaMalloc, no allocating
 * library routine); it clears the part of the scratch it uses, on `stream`,
 * before its kernel runs.
 *
 * The first call on each device looks up the scratch array's device address
 * (with that device current) and caches it; make that first call before any
 * stream capture on the device. A device reset (cudaDeviceReset) creates a
 * new context: the next call looks the address up again, and it too must
 * come before any capture. All calls share the one array: calls that may
 * overlap on the GPU (different streams, or graph replays running
 * concurrently) race on it and must be serialised by the caller. Such a
 * race gives wrong sets, never an access outside the array: a CTA whose
 * ticket lies past its own grid sets SPA_DEV_SCRATCH_RACE and stops.
 * ---------------------------------------------------------------------- */
int spa_build_kv_sets_noalloc(const int32_t* pos, int32_t n_queries, int32_t window, int32_t ratio,
                              const int32_t* topk, int32_t topk_width, int32_t* indptr,
                              int32_t* indices, int64_t capacity, uint32_t* dev_status,
                              spa_stream_t stream);

/* ------------------------------------------------------------------------
 * 2. spa_dequant_fp8_pages -- mixed FP8/BF16 cache: FP8 pages to BF16.
 *
 * Defined by "Roadmap item 24", section "Reuse and arithmetic" (a mixed
 * FP8/BF16 cache decoder with an explicit OCP/FNUZ format and 64/128-token
 * pages). Format: OCP E4M3 (bias 7, subnormals, S.1111.111 = NaN, max 448),
 * one FP32 scale per 64 consecutive elements of a token row.
 *
 * For every listed page pg and every element e of its rows:
 *   dst[pg][s][e] = bf16_rne( float(e4m3(src[pg][s][e])) * scales[pg][s][e/64] )
 * (one binary32 multiply, then round-to-nearest-even to BF16). Unlisted
 * pages of dst are not written.
 *
 * src       uint8 [num_pages, page_size, head_dim], 16-byte aligned
 * scales    float [num_pages, page_size, head_dim/64]
 * page_ids  int32 [n_page_ids]; ids outside [0, num_pages) set
 *           SPA_DEV_BAD_PAGE and are skipped
 * fp8_format 0 = OCP E4M3, 1 = E4M3 FNUZ (exponent bias 8, no -0, the
 *            code 0x80 is the NaN, largest magnitude 240)
 * dst       BF16 bits [num_pages, page_size, head_dim], 16-byte aligned
 * head_dim  a multiple of 64
 * ---------------------------------------------------------------------- */
int spa_dequant_fp8_pages(const uint8_t* src, const float* scales, int64_t num_pages,
                          int32_t page_size, int32_t head_dim, const int32_t* page_ids,
                          int32_t n_page_ids, int32_t fp8_format, uint16_t* dst,
                          uint32_t* dev_status, spa_stream_t stream);

/* ------------------------------------------------------------------------
 * 3. spa_sparse_sink_attn_fwd -- attention over the per-token sets.
 *
 * Defined by "Roadmap item 24", section "Reuse and arithmetic" (compressed
 * KV + full recent window + sink share the denominator; the sink has no V;
 * BF16 P/O and FP32 natural-log LSE), and "test: add block-level
 * DeepSeek-V4 attention test", "What this test actually drives" (sparse
 * decode over KV splits followed by a reduce: here an exact LSE merge).
 *
 * For query i (request b = req[i]) and head h, over the keys of set i:
 *   s_j   = scale * dot(q[i][h], k_j)
 *   LSE   = ln( e^{sink[h]} + sum_j e^{s_j} )
 *   O     = sum_j e^{s_j - LSE} v_j        (the sink contributes no V)
 * A window key (SPA_WINDOW_TAG | t) reads row t of request b through
 * pt_raw: page = pt_raw[b][t / raw_page_size], slot = t % raw_page_size;
 * a compressed key g reads row g through pt_cmp the same way. P is rounded
 * to BF16 before the PV product, as on the page; accumulation is FP32.
 * sink == NULL means no sink (plain softmax); an empty set gives O = 0 and
 * LSE = sink[h] (or -inf without a sink).
 *
 * q          BF16 [n_queries, num_heads, head_dim]; element (i,h,e) at
 *            q + i*q_stride_tok + h*q_stride_head + e. Base and both
 *            strides (in bytes) must be multiples of 16.
 * head_dim   64, 128 or 512 (d_qk = d_v). 512 is the DSV4-Flash attention
 *            shape ("Roadmap item 24", section "Reuse and arithmetic": the
 *            fixed H32 launch recipe; the 512-wide rows of the packed cache,
 *            decoded by spa_unpack_d512_pages): 32 heads per CTA, the
 *            products transposed (keys, then columns of d, on the tensor
 *            cores' M side); slices merge inside a cluster only, so
 *            num_splits is at most 8, no workspace is used, and 0 picks
 *            spa_sparse_sink_attn_choose_splits_d512(n, H)
 * num_heads  1..128, or a multiple of 128 (head_dim 64, 128); 1..32, or a
 *            multiple of 32 (head_dim 512)
 * k_raw, v_raw   BF16 [raw_num_pages, raw_page_size, head_dim], 16-B aligned
 * pt_raw     int32 [n_requests, pt_raw_cols]
 * k_cmp, v_cmp, pt_cmp   the compressed pool, laid out the same way; may be
 *            NULL when no set holds a compressed key (ratio 0)
 * page sizes powers of two, 1 .. 1024
 * req        int32 [n_queries]
 * indptr, indices   CSR key sets (as built by spa_build_kv_sets; any order
 *            within a set is accepted)
 * sink       float [num_heads] natural-log logits, or NULL
 * scale      > 0
 * out        BF16 [n_queries, num_heads, head_dim] contiguous, 16-B aligned
 * lse        float [n_queries, num_heads]
 * num_splits 0 = automatic (spa_sparse_sink_attn_choose_splits(n, H, 0)),
 *            1 = one CTA per query, S in 2..16 = the set of each query is
 *            cut into S slices of 64-key tiles whose partial results are
 *            merged exactly (O_s, LSE_s weighted by e^{LSE_s-LSE}).
 *            choose_splits: 1 for batches that fill the GPU; for small
 *            batches (decode) up to 4 slices, no more than fill one wave of
 *            CTAs; for a known long largest set, slices of >= 1024 keys.
 * workspace  >= spa_sparse_sink_attn_workspace_size(...) bytes for the same
 *            arguments: 0 bytes unsplit or with at most 8 slices (the slices
 *            of a query then run as one thread-block cluster and merge
 *            through distributed shared memory); 9..16 slices write FP32
 *            partial results there, merged by the last slice to finish.
 * ---------------------------------------------------------------------- */
size_t spa_sparse_sink_attn_workspace_size(int32_t n_queries, int32_t num_heads,
                                           int32_t head_dim, int32_t num_splits);
int spa_sparse_sink_attn_choose_splits(int32_t n_queries, int32_t num_heads,
                                       int32_t max_set_size);
/* head_dim 512: slices per query (1, 2, 4 or 8) so that one wave of CTAs, one
 * per SM, covers the batch; 1 once the batch fills the GPU. */
int spa_sparse_sink_attn_choose_splits_d512(int32_t n_queries, int32_t num_heads);
int spa_sparse_sink_attn_fwd(
    const uint16_t* q, int64_t q_stride_tok, int64_t q_stride_head, int32_t n_queries,
    int32_t num_heads, int32_t head_dim,
    const uint16_t* k_raw, const uint16_t* v_raw, int64_t raw_num_pages, int32_t raw_page_size,
    const int32_t* pt_raw, int32_t pt_raw_cols,
    const uint16_t* k_cmp, const uint16_t* v_cmp, int64_t cmp_num_pages, int32_t cmp_page_size,
    const int32_t* pt_cmp, int32_t pt_cmp_cols,
    const int32_t* req, int32_t n_requests, const int32_t* indptr, const int32_t* indices,
    const float* sink, float scale, uint16_t* out, float* lse, int32_t num_splits,
    void* workspace, size_t workspace_bytes, uint32_t* dev_status, spa_stream_t stream);

/* ------------------------------------------------------------------------
 * 3a. spa_sparse_sink_attn_fwd_inline_sets -- spa_sparse_sink_attn_fwd over
 * the sets spa_build_kv_sets builds, built inside the attention kernel from
 * the builder's own inputs (positions, top-k rows, W, ratio) instead of read
 * from CSR arrays.
 *
 * Same sets as section 1 ("Roadmap item 24", "Contracts and lifetime"; the
 * block-level test's layer types and its "Validation" rule on top-k): for
 * query i at position p = pos[i] and G = floor((p+1)/ratio),
 *   groups = none (ratio 0); { g : 0 <= g < G } (topk == NULL);
 *            { topk[i][j] : 0 <= topk[i][j] < G }, repeats removed (else)
 *   set_i  = ascending(groups U { SPA_WINDOW_TAG | t : max(0, p-W+1) <= t <= p })
 * The keys and their order are those of spa_build_kv_sets, so O and LSE are
 * bit-identical to spa_build_kv_sets followed by spa_sparse_sink_attn_fwd
 * with the same num_splits. In the decode timeline of the block-level test
 * the set build precedes the core; here it costs no launch and no round
 * trip through indptr/indices. A top-k row is reduced to its sorted groups
 * by the kernel's resolver warp once per (query, slice) unit.
 *
 * Arguments as for spa_sparse_sink_attn_fwd, without indptr/indices, plus:
 * pos        int32 [n_queries], 0 <= pos < 2^30 (else SPA_DEV_BAD_INDEX and
 *            an empty set for that query)
 * topk       int32 [n_queries, topk_width] row-major, 4-byte aligned, or
 *            NULL; entries < 0 (and those >= G) pick nothing. Ignored when
 *            ratio = 0.
 * topk_width 0 <= topk_width <= 512 (wider rows: SPA_ERR_UNSUPPORTED; build
 *            them with spa_build_kv_sets)
 * window     W >= 1
 * ratio      0, 4 or 128; ratio > 0 needs the compressed pool (k_cmp, v_cmp,
 *            pt_cmp non-NULL)
 * ---------------------------------------------------------------------- */
int spa_sparse_sink_attn_fwd_inline_sets(
    const uint16_t* q, int64_t q_stride_tok, int64_t q_stride_head, int32_t n_queries,
    int32_t num_heads, int32_t head_dim,
    const uint16_t* k_raw, const uint16_t* v_raw, int64_t raw_num_pages, int32_t raw_page_size,
    const int32_t* pt_raw, int32_t pt_raw_cols,
    const uint16_t* k_cmp, const uint16_t* v_cmp, int64_t cmp_num_pages, int32_t cmp_page_size,
    const int32_t* pt_cmp, int32_t pt_cmp_cols,
    const int32_t* req, int32_t n_requests, const int32_t* pos,
    const int32_t* topk, int32_t topk_width, int32_t window, int32_t ratio,
    const float* sink, float scale, uint16_t* out, float* lse, int32_t num_splits,
    void* workspace, size_t workspace_bytes, uint32_t* dev_status, spa_stream_t stream);

/* ------------------------------------------------------------------------
 * 3b. spa_sparse_sink_attn_fwd_fp8 -- the same attention over a mixed
 * cache whose compressed pool is stored in FP8, decoded inside the gather.
 *
 * Defined by "Roadmap item 24", section "Reuse and arithmetic" (the mixed
 * FP8/BF16 cache, an explicit OCP format, FP32 scales, decoded to BF16
 * before the BF16 attention). Every compressed element enters the products
 * as bf16_rne(float(e4m3) * scale), the value spa_dequant_fp8_pages writes,
 * so the result is bit-identical to decoding the pages first and calling
 * spa_sparse_sink_attn_fwd on the decoded pool.
 *
 * Arguments as for spa_sparse_sink_attn_fwd, except the compressed pool:
 * k_cmp_fp8, v_cmp_fp8    E4M3 codes [cmp_num_pages, cmp_page_size,
 *                         head_dim] bytes, 16-B aligned
 * k_cmp_scale, v_cmp_scale FP32 [cmp_num_pages, cmp_page_size,
 *                         head_dim / 64]: one scale per 64 elements
 * pt_cmp                  required (non-NULL)
 * fp8_format              0 = OCP E4M3, 1 = E4M3 FNUZ
 * The window (raw) pool stays BF16.
 * ---------------------------------------------------------------------- */
int spa_sparse_sink_attn_fwd_fp8(
    const uint16_t* q, int64_t q_stride_tok, int64_t q_stride_head, int32_t n_queries,
    int32_t num_heads, int32_t head_dim,
    const uint16_t* k_raw, const uint16_t* v_raw, int64_t raw_num_pages, int32_t raw_page_size,
    const int32_t* pt_raw, int32_t pt_raw_cols,
    const uint8_t* k_cmp_fp8, const uint8_t* v_cmp_fp8, const float* k_cmp_scale,
    const float* v_cmp_scale, int64_t cmp_num_pages, int32_t cmp_page_size,
    const int32_t* pt_cmp, int32_t pt_cmp_cols, int32_t fp8_format,
    const int32_t* req, int32_t n_requests, const int32_t* indptr, const int32_t* indices,
    const float* sink, float scale, uint16_t* out, float* lse, int32_t num_splits,
    void* workspace, size_t workspace_bytes, uint32_t* dev_status, spa_stream_t stream);

/* spa_sparse_sink_attn_fwd_fp8_inline_sets -- spa_sparse_sink_attn_fwd_fp8
 * over the sets of section 3a, built inside the kernel: the arguments of
 * spa_sparse_sink_attn_fwd_fp8 with indptr/indices replaced by pos, topk,
 * topk_width, window and ratio (meaning, limits and errors as in 3a). O and
 * LSE are bit-identical to spa_build_kv_sets followed by
 * spa_sparse_sink_attn_fwd_fp8 with the same num_splits. */
int spa_sparse_sink_attn_fwd_fp8_inline_sets(
    const uint16_t* q, int64_t q_stride_tok, int64_t q_stride_head, int32_t n_queries,
    int32_t num_heads, int32_t head_dim,
    const uint16_t* k_raw, const uint16_t* v_raw, int64_t raw_num_pages, int32_t raw_page_size,
    const int32_t* pt_raw, int32_t pt_raw_cols,
    const uint8_t* k_cmp_fp8, const uint8_t* v_cmp_fp8, const float* k_cmp_scale,
    const float* v_cmp_scale, int64_t cmp_num_pages, int32_t cmp_page_size,
    const int32_t* pt_cmp, int32_t pt_cmp_cols, int32_t fp8_format,
    const int32_t* req, int32_t n_requests, const int32_t* pos,
    const int32_t* topk, int32_t topk_width, int32_t window, int32_t ratio,
    const float* sink, float scale, uint16_t* out, float* lse, int32_t num_splits,
    void* workspace, size_t workspace_bytes, uint32_t* dev_status, spa_stream_t stream);

/* ------------------------------------------------------------------------
 * 3c. spa_sparse_sink_attn_bwd -- gradients of the attention with sink.
 *
 * The follow-on item of "Roadmap item 24 - joint compressed/window attention
 * with sink": dQ, dK/dV scattered to the pages, and d_sink, from the saved O
 * and LSE. With p_j = exp(scale q.k_j - LSE) recomputed per (query, head),
 * D = dO . O, ds_j = p_j (dO . v_j - D):
 *   dq += scale sum_j ds_j k_j         dk[row(j)] += scale ds_j q  (all heads)
 *   dv[row(j)] += p_j dO (all heads)   dsink[h] += -exp(sink_h - LSE) D
 * P and dS enter the tensor-core products as BF16; every sum is FP32.
 *
 * Arguments as for spa_sparse_sink_attn_fwd (BF16 pools only), plus:
 * out, lse   the forward's O (BF16 [n_queries, num_heads, head_dim],
 *            contiguous, 16-B aligned) and LSE (FP32 [n_queries, num_heads])
 * dout       dO, BF16 [n_queries, num_heads, head_dim], contiguous, 16-B aligned
 * dq         FP32 [n_queries, num_heads, head_dim], 16-B aligned
 * dk_raw, dv_raw  FP32 [raw_num_pages * raw_page_size, head_dim], 16-B
 *            aligned: the raw pools' gradient rows; dk_cmp, dv_cmp likewise
 *            for the compressed pool (required when pt_cmp is set)
 * dsink      FP32 [num_heads] or NULL (ignored when sink is NULL)
 * Every gradient is ADDED into its array (zero them for a fresh gradient);
 * the additions are FP32 atomics, so their order, and the last bits of a
 * sum, vary from run to run. Rows of faulty keys receive nothing (the
 * status word says why, as in the forward). num_splits as in the forward
 * (0 = automatic); slices add their dq. No workspace.
 * ---------------------------------------------------------------------- */
int spa_sparse_sink_attn_bwd(
    const uint16_t* q, int64_t q_stride_tok, int64_t q_stride_head, int32_t n_queries,
    int32_t num_heads, int32_t head_dim,
    const uint16_t* k_raw, const uint16_t* v_raw, int64_t raw_num_pages, int32_t raw_page_size,
    const int32_t* pt_raw, int32_t pt_raw_cols,
    const uint16_t* k_cmp, const uint16_t* v_cmp, int64_t cmp_num_pages, int32_t cmp_page_size,
    const int32_t* pt_cmp, int32_t pt_cmp_cols,
    const int32_t* req, int32_t n_requests, const int32_t* indptr, const int32_t* indices,
    const float* sink, float scale, const uint16_t* out, const float* lse, const uint16_t* dout,
    float* dq, float* dk_raw, float* dv_raw, float* dk_cmp, float* dv_cmp, float* dsink,
    int32_t num_splits, uint32_t* dev_status, spa_stream_t stream);

/* ------------------------------------------------------------------------
 * 4. spa_paged_kv_write -- new raw tokens into the paged window cache.
 *
 * Defined by "test: add block-level DeepSeek-V4 attention test", decode
 * kernel timeline and notes (the paged KV write, "swa_write" / "kvw_paged",
 * runs ahead of the sparse attention core); without the qk-norm and RoPE
 * the model fuses into it. Token j, of request b = req[j] at position
 * t = pos[j], is copied to row pt[b][t / page_size] * page_size +
 * t % page_size of k_pool and of v_pool.
 *
 * k_new, v_new  BF16 [n_tokens, head_dim] contiguous, 16-B aligned
 * head_dim      a multiple of 8
 * req, pos      int32 [n_tokens]; a request outside [0, n_requests) or a
 *               position outside the table sets SPA_DEV_BAD_INDEX, a page id
 *               outside [0, num_pages) SPA_DEV_BAD_PAGE; the token is skipped
 * pt            int32 [n_requests, pt_cols] (the raw page table)
 * page_size     power of two, 1 .. 1024
 * k_pool, v_pool BF16 [num_pages, page_size, head_dim], 16-B aligned
 * Rows not named by a token are left as they are; two tokens naming the
 * same row leave one of them there (which one is unspecified).
 * ---------------------------------------------------------------------- */
int spa_paged_kv_write(const uint16_t* k_new, const uint16_t* v_new, int32_t n_tokens, int32_t head_dim,
                       const int32_t* req, const int32_t* pos, const int32_t* pt, int32_t pt_cols,
                       int32_t n_requests, int32_t page_size, int64_t num_pages, uint16_t* k_pool,
                       uint16_t* v_pool, uint32_t* dev_status, spa_stream_t stream);

/* ------------------------------------------------------------------------
 * 5. spa_unpack_d512_pages -- packed 512-wide rows (584 bytes per token)
 * to BF16.
 *
 * "Roadmap item 24 - joint compressed/window attention with sink", review
 * notes on the packed joint KV gather: 584 bytes per token for a 512-wide
 * head, 576 of them data. Read as: bytes 0..447 OCP E4M3 codes (elements
 * 0..447), bytes 448..575 BF16 (elements 448..511), bytes 576..582 UE8M0
 * scales (2^(byte-127), one per 64 codes; 0xFF is NaN), byte 583 unused.
 * Element e < 448 -> bf16_rne(float(e4m3) * 2^(s-127)); the rest copied.
 *
 * src        uint8 [num_pages, page_size, 584], 8-B aligned
 * page_ids   int32 [n_page_ids]: the pages to decode; an id outside
 *            [0, num_pages) sets SPA_DEV_BAD_PAGE and that page is skipped
 * dst        BF16 [num_pages, page_size, 512], 16-B aligned; pages not
 *            listed are left untouched
 * page_size  1 .. 4096
 * ---------------------------------------------------------------------- */
int spa_unpack_d512_pages(const uint8_t* src, int64_t num_pages, int32_t page_size, const int32_t* page_ids,
                          int32_t n_page_ids, uint16_t* dst, uint32_t* dev_status, spa_stream_t stream);

/* ------------------------------------------------------------------------
 * Testing hook -- not part of the method.
 *
 * Every wait between the warp roles of the attention forward gives up after
 * a limit (1 s), sets SPA_DEV_TIMEOUT and lets the kernel unwind, so that a
 * stuck pipeline ends the call instead of hanging the GPU. The waits that
 * keep a CTA's memory alive until its own copies and tensor-core products
 * have finished always keep the 1 s limit.
 *
 * spa_testing_stall_attention(limit_ns) with limit_ns > 0 makes the forward
 * launches that follow (both head-width kernels; process-wide, every
 * device) wait, in every CTA, on a barrier that nothing ever arrives at,
 * with limit_ns as the limit of every wait between the roles: each CTA
 * times out there and unwinds, and the call returns with SPA_DEV_TIMEOUT
 * set and poisoned outputs. That is how the tests reach the timeout path
 * without a fault. limit_ns = 0 restores normal launches.
 * ---------------------------------------------------------------------- */
void spa_testing_stall_attention(uint64_t limit_ns);

#ifdef __cplusplus
}
#endif
#endif /* SPA_H_ */
