// FP8 (OCP E4M3, or E4M3 FNUZ) pages with one FP32 scale per 64 elements
// -> BF16 pages.
//
// Page "Roadmap item 24 - joint compressed/window attention with sink",
// section "Reuse and arithmetic": the mixed FP8/BF16 cache is decoded with
// an explicit format (OCP or FNUZ E4M3), in 64/128-token pages. Every
// element becomes bf16_rne(float(e4m3(byte)) * scale): the E4M3 -> half
// conversion is exact (every E4M3 value is a half value), half -> float is
// exact, then one binary32 multiply and one round-to-nearest-even to BF16.
//
// One CTA per listed page; each thread moves 16 source bytes (one 16-byte
// load) to 32 destination bytes (two 16-byte stores). HBM-bound: 3 bytes of
// traffic per element plus 4 bytes of scale per 64 elements.
#include "spa_device.cuh"
#include "spa_internal.h"

namespace spa {
namespace {

template <bool kFnuz>
__global__ void __launch_bounds__(256)
dequant_fp8_pages_kernel(const uint8_t* __restrict__ src, const float* __restrict__ scales,
                         int64_t num_pages, int32_t chunks_per_page,
                         const int32_t* __restrict__ page_ids, uint16_t* __restrict__ dst,
                         uint32_t* dev_status) {
  const int64_t pg = page_ids[blockIdx.x];
  if (pg < 0 || pg >= num_pages) {
    if (threadIdx.x == 0) report(dev_status, SPA_DEV_BAD_PAGE);
    return;
  }
  const int64_t page_elem0 = pg * static_cast<int64_t>(chunks_per_page) * 16;
  for (int32_t c = threadIdx.x; c < chunks_per_page; c += blockDim.x) {
    const int64_t e0 = page_elem0 + static_cast<int64_t>(c) * 16;
    const uint4 raw = __ldg(reinterpret_cast<const uint4*>(src + e0));
    const float s = __ldg(scales + (e0 >> 6));  // rows are whole multiples of 64
    uint32_t o[8];
    decode_e4m3x16<kFnuz>(raw, s, o);
    uint4* out = reinterpret_cast<uint4*>(dst + e0);
    out[0] = make_uint4(o[0], o[1], o[2], o[3]);
    out[1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

}  // namespace

cudaError_t launch_dequant_fp8_pages(const uint8_t* src, const float* scales, int64_t num_pages,
                                     int32_t page_size, int32_t head_dim, const int32_t* page_ids,
                                     int32_t n_page_ids, bool fnuz, uint16_t* dst, uint32_t* dev_status,
                                     cudaStream_t stream) {
  if (n_page_ids == 0) return cudaSuccess;
  const int32_t chunks = page_size * (head_dim / 16);
  const int threads = chunks >= 256 ? 256 : ((chunks + 31) / 32) * 32;
  if (fnuz)
    dequant_fp8_pages_kernel<true><<<static_cast<unsigned>(n_page_ids), threads, 0, stream>>>(
        src, scales, num_pages, chunks, page_ids, dst, dev_status);
  else
    dequant_fp8_pages_kernel<false><<<static_cast<unsigned>(n_page_ids), threads, 0, stream>>>(
        src, scales, num_pages, chunks, page_ids, dst, dev_status);
  return cudaGetLastError();
}

}  // namespace spa
