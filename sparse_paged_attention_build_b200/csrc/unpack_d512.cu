// Packed 512-wide rows (584 bytes per token) -> BF16 pages.
//
// Page "Roadmap item 24 - joint compressed/window attention with sink",
// review notes on the packed joint KV gather: a 512-wide head is stored in
// 584 bytes per token, 576 of them data. Read here as 448 OCP E4M3 codes
// (elements 0..447), 64 BF16 values (elements 448..511, 128 bytes), then 7
// UE8M0 scale bytes (2^(byte-127), one per 64 codes) and one unused byte.
// Element e < 448 becomes bf16_rne(float(e4m3) * 2^(s-127)) (one binary32
// multiply, exact unless the product is subnormal, then the same rounding
// as the oracle's); the BF16 tail is copied.
//
// One CTA per listed page; an item is 16 codes (32 output bytes) or 16 BF16
// tail values, 32 items per token. A token's 584 bytes start on an 8-byte
// boundary only, so the loads are 8-byte vectors (a warp still covers whole
// 32-byte sectors); the stores are 16-byte vectors. HBM-bound: 584 bytes
// read and 1024 written per token.
#include "spa_device.cuh"
#include "spa_internal.h"

namespace spa {
namespace {

constexpr int kRowBytes = 584;
constexpr int kCodes = 448;
constexpr int kItemsPerRow = kCodes / 16 + 4;   // 28 code items, 4 tail items

__device__ __forceinline__ float ue8m0_scale(uint32_t b) {
  if (b == 0xFFu) return __int_as_float(0x7fffffff);
  if (b == 0u) return __int_as_float(0x00400000);   // 2^-127, a subnormal
  return __int_as_float(static_cast<int>(b << 23));
}

__global__ void __launch_bounds__(256)
unpack_d512_kernel(const uint8_t* __restrict__ src, int64_t num_pages, int32_t page_size,
                   const int32_t* __restrict__ page_ids, uint16_t* __restrict__ dst, uint32_t* dev_status) {
  const int64_t pg = page_ids[blockIdx.x];
  if (pg < 0 || pg >= num_pages) {
    if (threadIdx.x == 0) report(dev_status, SPA_DEV_BAD_PAGE);
    return;
  }
  const int32_t items = page_size * kItemsPerRow;
  for (int32_t q = threadIdx.x; q < items; q += blockDim.x) {
    const int64_t row = pg * page_size + q / kItemsPerRow;
    const int m = q % kItemsPerRow;
    const uint8_t* in = src + row * kRowBytes;
    uint4* out = reinterpret_cast<uint4*>(dst + row * 512);
    if (m < kCodes / 16) {
      const uint2 a = __ldg(reinterpret_cast<const uint2*>(in + 16 * m));
      const uint2 b = __ldg(reinterpret_cast<const uint2*>(in + 16 * m + 8));
      const float s = ue8m0_scale(__ldg(in + kCodes + 128 + (m >> 2)));
      uint32_t o[8];
      decode_e4m3x16<false>(make_uint4(a.x, a.y, b.x, b.y), s, o);
      out[2 * m] = make_uint4(o[0], o[1], o[2], o[3]);
      out[2 * m + 1] = make_uint4(o[4], o[5], o[6], o[7]);
    } else {
      const int k = m - kCodes / 16;
      const uint2* t = reinterpret_cast<const uint2*>(in + kCodes + 32 * k);
      const uint2 a = __ldg(t), b = __ldg(t + 1), c = __ldg(t + 2), d = __ldg(t + 3);
      out[56 + 2 * k] = make_uint4(a.x, a.y, b.x, b.y);
      out[56 + 2 * k + 1] = make_uint4(c.x, c.y, d.x, d.y);
    }
  }
}

}  // namespace

cudaError_t launch_unpack_d512_pages(const uint8_t* src, int64_t num_pages, int32_t page_size,
                                     const int32_t* page_ids, int32_t n_page_ids, uint16_t* dst,
                                     uint32_t* dev_status, cudaStream_t stream) {
  if (n_page_ids == 0) return cudaSuccess;
  const int32_t items = page_size * kItemsPerRow;
  const int threads = items >= 256 ? 256 : ((items + 31) / 32) * 32;
  unpack_d512_kernel<<<static_cast<unsigned>(n_page_ids), threads, 0, stream>>>(src, num_pages, page_size,
                                                                                page_ids, dst, dev_status);
  return cudaGetLastError();
}

}  // namespace spa
