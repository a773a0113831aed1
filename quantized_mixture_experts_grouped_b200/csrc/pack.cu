// Symmetric group-128 int4 quantiser + packer ("Every Expert Counts: ExactMoE for
// Memory-Efficient W4A16 Inference", Abstract: group-128 four-bit weights for the routed
// experts only). One CTA quantises 128 rows x one 128-K group: it stages the bf16 values in shared
// memory with coalesced 32-bit loads, then each thread owns one row: absmax, scale, codes, and
// four 16-byte pieces written in the "MW4T v2" layout (row r lands in the 512-byte chunk of its
// 8-row group and K group; eight consecutive rows fill 128 contiguous bytes per quarter).
#include "common.cuh"

namespace moe {
namespace {

constexpr int kRowWords = kGroup / 2;      // 64 words of bf16 pairs per row of the tile
constexpr int kRowPitch = kRowWords + 1;   // odd pitch: thread r reading word w hits bank (r+w)%32

__global__ void __launch_bounds__(128) quantize_pack_kernel(const uint16_t* __restrict__ w, int N, int K,
                                                            uint8_t* __restrict__ packed,
                                                            uint16_t* __restrict__ scales) {
  __shared__ uint32_t tile[kRowBlock * kRowPitch];
  const int g = blockIdx.x, rb = blockIdx.y, e = blockIdx.z;
  const int G = K / kGroup;
  const int tid = threadIdx.x;
  const uint32_t* src = reinterpret_cast<const uint32_t*>(w + ((size_t)e * N + (size_t)rb * kRowBlock) * K +
                                                          (size_t)g * kGroup);
  const size_t row_words = (size_t)K / 2;
  for (int i = tid; i < kRowBlock * kRowWords; i += blockDim.x) {
    const int r = i / kRowWords, c = i % kRowWords;
    tile[r * kRowPitch + c] = __ldg(src + r * row_words + c);
  }
  __syncthreads();

  const int r = tid;
  const uint32_t* row = tile + r * kRowPitch;
  float a = 0.f;
  for (int c = 0; c < kRowWords; ++c) {
    const uint32_t v = row[c];
    a = fmaxf(a, fabsf(bf16_bits_to_float(v & 0xffffu)));
    a = fmaxf(a, fabsf(bf16_bits_to_float(v >> 16)));
  }
  const float s32 = a / 7.0f;                       // IEEE fp32 division (no fast-math)
  const __nv_bfloat16 sb = __float2bfloat16_rn(s32);
  const float sf = __bfloat162float(sb);

  const size_t chunk = ((size_t)rb * (kRowBlock / kRowGroup) + r / kRowGroup) * G + g;
  uint8_t* dst = packed + (size_t)e * ((size_t)N * K / 2) + chunk * kChunkBytes + (size_t)(r % kRowGroup) * 16;
  for (int kq = 0; kq < 4; ++kq) {
    uint32_t words[4];
    for (int wi = 0; wi < 4; ++wi) {
      uint32_t word = 0;
      for (int el = 0; el < 8; ++el) {
        const int kk = kq * 32 + wi * 8 + el;
        const uint32_t pair = row[kk >> 1];
        const float v = bf16_bits_to_float((kk & 1) ? (pair >> 16) : (pair & 0xffffu));
        int q = 0;
        if (sf != 0.f) q = (int)fminf(7.f, fmaxf(-8.f, rintf(v / sf)));
        word |= (uint32_t)(q + 8) << (16 * (el & 1) + 4 * (el >> 1));
      }
      words[wi] = word;
    }
    *reinterpret_cast<uint4*>(dst + kq * 128) = make_uint4(words[0], words[1], words[2], words[3]);
  }
  scales[(size_t)e * ((size_t)N * G) + chunk * kRowGroup + r % kRowGroup] = __bfloat16_as_ushort(sb);
}

}  // namespace

int launch_quantize_pack(const uint16_t* w, int E, int N, int K, uint8_t* packed, uint16_t* scales,
                         cudaStream_t s) {
  if (E == 0) return MOE_OK;
  dim3 grid(K / kGroup, N / kRowBlock, E);
  quantize_pack_kernel<<<grid, 128, 0, s>>>(w, N, K, packed, scales);
  return check_launch("quantize_pack_kernel");
}

}  // namespace moe
