// CUDA-core grouped W4A16 MoE FFN and the shared combine ("Every Expert Counts: ExactMoE for
// Memory-Efficient W4A16 Inference", Abstract: every selected expert runs, grouped by expert).
//
// This path favours plainness over speed and serves as the on-device reference of the
// optimised paths: pairs are grouped by expert (moe_permute), rows gathered, then
//   gate/up : one thread per output feature i, a tile of 8 pairs of one expert, exact fp32
//             dequantisation q*s, fp32 FMA; h = silu(g) * u rounded to bf16;
//   down    : one thread per output row n, same tiling, fp32 result per pair;
//   combine : out[t] = sum_j wts[t][j] * y_pair(t, j) in fixed j order (fp32), bf16 out.
#include "common.cuh"

namespace moe {
namespace {

constexpr int kPairsPerTile = 8;

// tiles[e] prefix (E+1 entries) of ceil(count_e / per_tile) over experts that are resident.
__global__ void __launch_bounds__(kMaxExperts) plan_tiles_kernel(const int32_t* __restrict__ counts, int E,
                                                                 const int32_t* __restrict__ table, int per_tile,
                                                                 int32_t* __restrict__ tile_prefix) {
  __shared__ int tot[kMaxExperts];
  const int e = threadIdx.x;
  int n = 0;
  if (e < E && slot_of(table, e) >= 0) n = (counts[e] + per_tile - 1) / per_tile;
  tot[e] = n;
  __syncthreads();
  for (int o = 1; o < kMaxExperts; o <<= 1) {
    const int v = (e >= o) ? tot[e - o] : 0;
    __syncthreads();
    tot[e] += v;
    __syncthreads();
  }
  if (e < E) tile_prefix[e] = tot[e] - n;
  if (e == E - 1) tile_prefix[E] = tot[e];
}

// Expert owning flattened tile `tile` (tile_prefix is non-decreasing); -1 past the end.
__device__ int find_tile_expert(const int32_t* tile_prefix, int E, int tile) {
  if (tile >= tile_prefix[E]) return -1;
  int lo = 0, hi = E - 1;
  while (lo < hi) {               // largest e with tile_prefix[e] <= tile
    const int mid = (lo + hi + 1) >> 1;
    if (tile_prefix[mid] <= tile) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Dequantises the 32 weights of one 16-byte chunk exactly: w = (code - 8) * s.
__device__ __forceinline__ void dequant32(uint4 c, float s, float* w) {
  const uint32_t words[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
  for (int wi = 0; wi < 4; ++wi)
#pragma unroll
    for (int el = 0; el < 8; ++el) {
      const int code = (words[wi] >> (16 * (el & 1) + 4 * (el >> 1))) & 0xF;
      w[wi * 8 + el] = (float)(code - 8) * s;
    }
}

struct TileInfo { int e, slot, p0, np; };

__device__ bool load_tile_info(const int32_t* tile_prefix, const int32_t* offsets, const int32_t* table, int E,
                               TileInfo* ti) {
  __shared__ TileInfo sh;
  if (threadIdx.x == 0) {
    const int e = find_tile_expert(tile_prefix, E, blockIdx.x);
    sh.e = e;
    if (e >= 0) {
      sh.slot = slot_of(table, e);
      sh.p0 = offsets[e] + (blockIdx.x - tile_prefix[e]) * kPairsPerTile;
      sh.np = min(kPairsPerTile, offsets[e + 1] - sh.p0);
    }
  }
  __syncthreads();
  *ti = sh;
  return sh.e >= 0;
}

__global__ void __launch_bounds__(128) gateup_simple_kernel(
    const uint16_t* __restrict__ xp, int H, int I, int E, const int32_t* __restrict__ tile_prefix,
    const int32_t* __restrict__ offsets, const int32_t* __restrict__ table, const uint8_t* __restrict__ w13,
    const uint16_t* __restrict__ s13, uint16_t* __restrict__ hp) {
  TileInfo ti;
  if (!load_tile_info(tile_prefix, offsets, table, E, &ti)) return;
  __shared__ float xs[kPairsPerTile][kGroup];
  const int r = threadIdx.x, ib = blockIdx.y;
  const int G = H / kGroup;
  const size_t wstride = (size_t)2 * I * H / 2, sstride = (size_t)2 * I * G;
  const int ng = ib * kRowBlock + r, nu = I + ng;   // gate and up rows of this thread
  const uint8_t* wg = w13 + ti.slot * wstride + chunk_offset(ng / kRowGroup, 0, G) + (ng % kRowGroup) * 16;
  const uint8_t* wu = w13 + ti.slot * wstride + chunk_offset(nu / kRowGroup, 0, G) + (nu % kRowGroup) * 16;
  const uint16_t* sg = s13 + ti.slot * sstride + chunk_scale_index(ng / kRowGroup, 0, G) + ng % kRowGroup;
  const uint16_t* su = s13 + ti.slot * sstride + chunk_scale_index(nu / kRowGroup, 0, G) + nu % kRowGroup;
  float ag[kPairsPerTile] = {}, au[kPairsPerTile] = {};
  for (int g = 0; g < G; ++g) {
    __syncthreads();
    for (int pp = 0; pp < kPairsPerTile; ++pp)
      xs[pp][r] = pp < ti.np ? bf16_bits_to_float(xp[(size_t)(ti.p0 + pp) * H + g * kGroup + r]) : 0.f;
    __syncthreads();
    const float scg = bf16_bits_to_float(sg[(size_t)g * kRowGroup]);
    const float scu = bf16_bits_to_float(su[(size_t)g * kRowGroup]);
    for (int kq = 0; kq < 4; ++kq) {
      float fg[32], fu[32];
      dequant32(*reinterpret_cast<const uint4*>(wg + (size_t)g * kChunkBytes + kq * 128), scg, fg);
      dequant32(*reinterpret_cast<const uint4*>(wu + (size_t)g * kChunkBytes + kq * 128), scu, fu);
#pragma unroll
      for (int c = 0; c < 32; ++c)
#pragma unroll
        for (int pp = 0; pp < kPairsPerTile; ++pp) {
          ag[pp] = fmaf(fg[c], xs[pp][kq * 32 + c], ag[pp]);
          au[pp] = fmaf(fu[c], xs[pp][kq * 32 + c], au[pp]);
        }
    }
  }
  const int i = ib * kRowBlock + r;
  for (int pp = 0; pp < ti.np; ++pp) {
    const float g = ag[pp];
    const float h = g / (1.f + expf(-g)) * au[pp];
    hp[(size_t)(ti.p0 + pp) * I + i] = __bfloat16_as_ushort(__float2bfloat16_rn(h));
  }
}

__global__ void __launch_bounds__(128) down_simple_kernel(
    const uint16_t* __restrict__ hp, int H, int I, int E, const int32_t* __restrict__ tile_prefix,
    const int32_t* __restrict__ offsets, const int32_t* __restrict__ table, const uint8_t* __restrict__ w2,
    const uint16_t* __restrict__ s2, float* __restrict__ yp) {
  TileInfo ti;
  if (!load_tile_info(tile_prefix, offsets, table, E, &ti)) return;
  __shared__ float hs[kPairsPerTile][kGroup];
  const int r = threadIdx.x, nb = blockIdx.y;
  const int G = I / kGroup;
  const size_t wstride = (size_t)H * I / 2, sstride = (size_t)H * G;
  const int n0 = nb * kRowBlock + r;
  const uint8_t* wd = w2 + ti.slot * wstride + chunk_offset(n0 / kRowGroup, 0, G) + (n0 % kRowGroup) * 16;
  const uint16_t* sd = s2 + ti.slot * sstride + chunk_scale_index(n0 / kRowGroup, 0, G) + n0 % kRowGroup;
  float acc[kPairsPerTile] = {};
  for (int g = 0; g < G; ++g) {
    __syncthreads();
    for (int pp = 0; pp < kPairsPerTile; ++pp)
      hs[pp][r] = pp < ti.np ? bf16_bits_to_float(hp[(size_t)(ti.p0 + pp) * I + g * kGroup + r]) : 0.f;
    __syncthreads();
    const float sc = bf16_bits_to_float(sd[(size_t)g * kRowGroup]);
    for (int kq = 0; kq < 4; ++kq) {
      float f[32];
      dequant32(*reinterpret_cast<const uint4*>(wd + (size_t)g * kChunkBytes + kq * 128), sc, f);
#pragma unroll
      for (int c = 0; c < 32; ++c)
#pragma unroll
        for (int pp = 0; pp < kPairsPerTile; ++pp) acc[pp] = fmaf(f[c], hs[pp][kq * 32 + c], acc[pp]);
    }
  }
  const int n = nb * kRowBlock + r;
  for (int pp = 0; pp < ti.np; ++pp) yp[(size_t)(ti.p0 + pp) * H + n] = acc[pp];
}

// out[t][n..n+8) = bf16( acc_in + sum_j wts[t][j] * yp[inv[t][j]][n..] ), skipped experts
// (slot -1) contributing nothing. acc (fp32 [T][H]) carries slot-cache waves.
__global__ void __launch_bounds__(256) combine_kernel(const float* __restrict__ yp, const int32_t* __restrict__ idx,
                                                      const float* __restrict__ wts, const int32_t* __restrict__ inv,
                                                      const int32_t* __restrict__ table, int H, int k,
                                                      float* __restrict__ acc, bool accumulate,
                                                      uint16_t* __restrict__ out) {
  const int t = blockIdx.x;
  const int n0 = (blockIdx.y * blockDim.x + threadIdx.x) * 8;
  if (n0 >= H) return;
  float v[8];
  float* accp = acc + (size_t)t * H + n0;
  if (accumulate) {
    const float4 a0 = *reinterpret_cast<const float4*>(accp), a1 = *reinterpret_cast<const float4*>(accp + 4);
    v[0] = a0.x; v[1] = a0.y; v[2] = a0.z; v[3] = a0.w; v[4] = a1.x; v[5] = a1.y; v[6] = a1.z; v[7] = a1.w;
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = 0.f;
  }
  for (int j = 0; j < k; ++j) {
    const int e = idx[(size_t)t * k + j];
    if (slot_of(table, e) < 0) continue;
    const float w = wts[(size_t)t * k + j];
    const float* y = yp + (size_t)inv[(size_t)t * k + j] * H + n0;
    const float4 y0 = *reinterpret_cast<const float4*>(y), y1 = *reinterpret_cast<const float4*>(y + 4);
    v[0] = fmaf(w, y0.x, v[0]); v[1] = fmaf(w, y0.y, v[1]); v[2] = fmaf(w, y0.z, v[2]); v[3] = fmaf(w, y0.w, v[3]);
    v[4] = fmaf(w, y1.x, v[4]); v[5] = fmaf(w, y1.y, v[5]); v[6] = fmaf(w, y1.z, v[6]); v[7] = fmaf(w, y1.w, v[7]);
  }
  if (out) {
    uint32_t pk[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __nv_bfloat162 b = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
      pk[i] = *reinterpret_cast<const uint32_t*>(&b);
    }
    *reinterpret_cast<uint4*>(out + (size_t)t * H + n0) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    if (accumulate) {
      *reinterpret_cast<float4*>(accp) = make_float4(0.f, 0.f, 0.f, 0.f);
      *reinterpret_cast<float4*>(accp + 4) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  } else {
    *reinterpret_cast<float4*>(accp) = make_float4(v[0], v[1], v[2], v[3]);
    *reinterpret_cast<float4*>(accp + 4) = make_float4(v[4], v[5], v[6], v[7]);
  }
}

}  // namespace

int launch_combine(const FfnArgs& a, const WsLayout& L, cudaStream_t s) {
  if (a.T == 0) return MOE_OK;
  dim3 grid(a.T, ceil_div(a.H, 256 * 8));
  combine_kernel<<<grid, 256, 0, s>>>(reinterpret_cast<const float*>(a.ws + L.yp), a.idx, a.wts,
                                      reinterpret_cast<const int32_t*>(a.ws + L.inv), a.slot, a.H, a.k,
                                      reinterpret_cast<float*>(a.ws + L.acc), a.accumulate, a.out);
  return check_launch("combine_kernel");
}

int ffn_simple(const FfnArgs& a, cudaStream_t s) {
  const WsLayout L = ws_layout(a.T, a.H, a.I, a.E, a.k);
  const int Tk = a.T * a.k;
  int32_t* counts = reinterpret_cast<int32_t*>(a.ws + L.counts);
  int32_t* offsets = reinterpret_cast<int32_t*>(a.ws + L.offsets);
  int32_t* perm = reinterpret_cast<int32_t*>(a.ws + L.perm);
  int32_t* inv = reinterpret_cast<int32_t*>(a.ws + L.inv);
  int32_t* tiles = reinterpret_cast<int32_t*>(a.ws + L.tiles);
  uint16_t* xp = reinterpret_cast<uint16_t*>(a.ws + L.xp);
  uint16_t* hp = reinterpret_cast<uint16_t*>(a.ws + L.hp);
  float* yp = reinterpret_cast<float*>(a.ws + L.yp);
  if (int rc = launch_permute(a.idx, a.T, a.k, a.E, counts, offsets, perm, inv,
                              reinterpret_cast<int32_t*>(a.ws + L.perm_scratch), s))
    return rc;
  plan_tiles_kernel<<<1, kMaxExperts, 0, s>>>(counts, a.E, a.slot, kPairsPerTile, tiles);
  if (int rc = check_launch("plan_tiles_kernel")) return rc;
  if (int rc = launch_gather_rows(a.x, perm, Tk, a.k, a.H, xp, s)) return rc;
  const int max_tiles = ceil_div(Tk, kPairsPerTile) + a.E;
  if (Tk > 0) {
    gateup_simple_kernel<<<dim3(max_tiles, a.I / kRowBlock), 128, 0, s>>>(xp, a.H, a.I, a.E, tiles, offsets, a.slot,
                                                                         a.w13, a.s13, hp);
    if (int rc = check_launch("gateup_simple_kernel")) return rc;
    down_simple_kernel<<<dim3(max_tiles, a.H / kRowBlock), 128, 0, s>>>(hp, a.H, a.I, a.E, tiles, offsets, a.slot,
                                                                       a.w2, a.s2, yp);
    if (int rc = check_launch("down_simple_kernel")) return rc;
  }
  return launch_combine(a, L, s);
}

}  // namespace moe
