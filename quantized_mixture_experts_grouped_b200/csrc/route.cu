// Top-k router and expert grouping ("Every Expert Counts: ExactMoE for Memory-Efficient W4A16
// Inference", Abstract: the BF16 router's top-k procedure is left unchanged and all selected
// experts run through fused grouped kernels).
//
// Router: one warp per token. Each logit becomes a 32-bit key (order-preserving image of the
// bf16 value in the high half, 0xffff - expert id in the low half), so one warp max-reduction
// (redux.sync) picks the largest logit and, among equal logits, the lowest id. k rounds give the
// top-k in order. Softmax in fp32 over all E, then renormalised over the k chosen.
//
// Grouping: a stable counting sort of the T*k pairs by expert in three small launches
// (per-chunk histogram, column scan, per-chunk stable placement with warp match + prefix).
#include "common.cuh"

namespace moe {

__device__ __forceinline__ uint32_t route_key(uint32_t bits, int e) {
  bits &= 0xffffu;
  if (bits == 0x8000u) bits = 0;                                  // -0 ties with +0
  const uint32_t ord = (bits & 0x8000u) ? (~bits & 0xffffu) : (bits | 0x8000u);
  return (ord << 16) | (0xffffu - (uint32_t)e);
}

namespace {

constexpr int kMaxPerLane = kMaxExperts / 32;

__global__ void __launch_bounds__(128) route_kernel(const uint16_t* __restrict__ logits, int T, int E, int k,
                                                    int32_t* __restrict__ idx, float* __restrict__ wts) {
  pdl_begin();
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (t >= T) return;
  const uint16_t* lt = logits + (size_t)t * E;
  uint32_t key[kMaxPerLane];
  float lv[kMaxPerLane];
  uint32_t taken = 0;
#pragma unroll
  for (int i = 0; i < kMaxPerLane; ++i) {
    const int e = lane + 32 * i;
    if (e < E) {
      const uint32_t b = lt[e];
      key[i] = route_key(b, e);
      lv[i] = bf16_bits_to_float(b);
    } else {
      key[i] = 0;
      lv[i] = -INFINITY;
    }
  }
  int chosen[kMaxPerLane];   // lane (j % 32) keeps choice j in chosen[j / 32]
  float mx = 0.f;
  for (int j = 0; j < k; ++j) {
    uint32_t best = 0;
#pragma unroll
    for (int i = 0; i < kMaxPerLane; ++i)
      if (!(taken >> i & 1u) && key[i] > best) best = key[i];
    const uint32_t win = __reduce_max_sync(0xffffffffu, best);
    const int e = 0xffff - (int)(win & 0xffffu);
    if ((e & 31) == lane) taken |= 1u << (e >> 5);
#pragma unroll
    for (int i = 0; i < kMaxPerLane; ++i)
      if (j == 32 * i + lane) chosen[i] = e;
    if (j == 0) {   // the largest logit, decoded back from its key
      const uint32_t ord = win >> 16;
      mx = bf16_bits_to_float((ord & 0x8000u) ? (ord & 0x7fffu) : (~ord & 0xffffu));
    }
  }
  float z = 0.f;
#pragma unroll
  for (int i = 0; i < kMaxPerLane; ++i)
    if (lane + 32 * i < E) z += expf(lv[i] - mx);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
  float p[kMaxPerLane];
  float sel = 0.f;
#pragma unroll
  for (int i = 0; i < kMaxPerLane; ++i) {
    p[i] = 0.f;
    if (32 * i + lane < k) p[i] = expf(bf16_bits_to_float(lt[chosen[i]]) - mx) / z;
    sel += p[i];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sel += __shfl_xor_sync(0xffffffffu, sel, o);
#pragma unroll
  for (int i = 0; i < kMaxPerLane; ++i) {
    const int j = 32 * i + lane;
    if (j < k) {
      idx[(size_t)t * k + j] = chosen[i];
      wts[(size_t)t * k + j] = p[i] / sel;
    }
  }
}

constexpr int kChunk = 1024;   // pairs per permute block

// scratch: chunk_counts [nb][E] then chunk_base [nb][E]
__global__ void __launch_bounds__(kChunk) perm_count_kernel(const int32_t* __restrict__ idx, int Tk, int E,
                                                            int32_t* __restrict__ chunk_counts) {
  pdl_begin();
  __shared__ int cnt[kMaxExperts];
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  const int p = blockIdx.x * kChunk + threadIdx.x;
  if (p < Tk) {
    const int e = idx[p];
    if ((unsigned)e < (unsigned)E) atomicAdd(&cnt[e], 1);   // out-of-range ids are dropped
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) chunk_counts[(size_t)blockIdx.x * E + e] = cnt[e];
}

__global__ void __launch_bounds__(kMaxExperts) perm_scan_kernel(int nb, int E, const int32_t* __restrict__ chunk_counts,
                                                                int32_t* __restrict__ chunk_base,
                                                                int32_t* __restrict__ counts,
                                                                int32_t* __restrict__ offsets) {
  pdl_begin();
  __shared__ int tot[kMaxExperts];
  const int e = threadIdx.x;
  int run = 0;
  if (e < E) {
    for (int b = 0; b < nb; ++b) {
      chunk_base[(size_t)b * E + e] = run;
      run += chunk_counts[(size_t)b * E + e];
    }
    counts[e] = run;
  }
  tot[e] = (e < E) ? run : 0;
  __syncthreads();
  // inclusive scan over experts (Hillis-Steele; E <= 256)
  for (int o = 1; o < kMaxExperts; o <<= 1) {
    const int v = (e >= o) ? tot[e - o] : 0;
    __syncthreads();
    tot[e] += v;
    __syncthreads();
  }
  const int excl = tot[e] - ((e < E) ? run : 0);
  if (e < E) {
    offsets[e] = excl;
    for (int b = 0; b < nb; ++b) chunk_base[(size_t)b * E + e] += excl;
  }
  if (e == E - 1) offsets[E] = tot[e];
}

__global__ void __launch_bounds__(kChunk) perm_place_kernel(const int32_t* __restrict__ idx, int Tk, int E,
                                                            const int32_t* __restrict__ chunk_base,
                                                            int32_t* __restrict__ perm, int32_t* __restrict__ inv) {
  pdl_begin();
  __shared__ int wcount[kChunk / 32][kMaxExperts];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < (kChunk / 32) * E; i += blockDim.x) wcount[i / E][i % E] = 0;
  __syncthreads();
  const int p = blockIdx.x * kChunk + threadIdx.x;
  int e = (p < Tk) ? idx[p] : -1;
  if ((unsigned)e >= (unsigned)E) e = -1;
  const unsigned same = __match_any_sync(0xffffffffu, e);
  const unsigned lower = same & ((1u << lane) - 1u);
  if (e >= 0 && lower == 0) wcount[warp][e] = __popc(same);
  __syncthreads();
  if (e >= 0) {
    int rank = __popc(lower);
    for (int w = 0; w < warp; ++w) rank += wcount[w][e];
    const int pos = chunk_base[(size_t)blockIdx.x * E + e] + rank;
    perm[pos] = p;
    inv[p] = pos;
  }
}

__global__ void gather_rows_kernel(const uint16_t* __restrict__ x, const int32_t* __restrict__ perm, int k, int H,
                                   uint16_t* __restrict__ xp) {
  pdl_begin();
  const int pos = blockIdx.x;
  const int t = perm[pos] / k;
  const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * H);
  uint4* dst = reinterpret_cast<uint4*>(xp + (size_t)pos * H);
  for (int i = threadIdx.x; i < H / 8; i += blockDim.x) dst[i] = __ldg(src + i);
}

}  // namespace

size_t permute_scratch_count(int T, int k, int E) {
  const int nb = ceil_div(T * k, kChunk);
  return (size_t)2 * nb * E;
}

int launch_route(const uint16_t* logits, int T, int E, int k, int32_t* idx, float* wts, cudaStream_t s) {
  if (T == 0) return MOE_OK;
  note_launch();
  return check_cuda(launch_pdl(route_kernel, dim3(ceil_div(T, 4)), dim3(128), 0, s, logits, T, E, k, idx, wts),
                    "route_kernel");
}

int launch_permute(const int32_t* idx, int T, int k, int E, int32_t* counts, int32_t* offsets, int32_t* perm,
                   int32_t* inv, int32_t* scratch, cudaStream_t s) {
  const int Tk = T * k;
  const int nb = ceil_div(Tk, kChunk);
  int32_t* chunk_counts = scratch;
  int32_t* chunk_base = scratch + (size_t)nb * E;
  if (nb > 0) {
    note_launch();
    if (int rc = check_cuda(launch_pdl(perm_count_kernel, dim3(nb), dim3(kChunk), 0, s, idx, Tk, E, chunk_counts),
                            "perm_count_kernel"))
      return rc;
  }
  note_launch();
  if (int rc = check_cuda(launch_pdl(perm_scan_kernel, dim3(1), dim3(kMaxExperts), 0, s, nb, E,
                                     (const int32_t*)chunk_counts, chunk_base, counts, offsets),
                          "perm_scan_kernel"))
    return rc;
  if (nb > 0) {
    note_launch();
    if (int rc = check_cuda(launch_pdl(perm_place_kernel, dim3(nb), dim3(kChunk), 0, s, idx, Tk, E,
                                       (const int32_t*)chunk_base, perm, inv),
                            "perm_place_kernel"))
      return rc;
  }
  return MOE_OK;
}

int launch_gather_rows(const uint16_t* x, const int32_t* perm, int Tk, int k, int H, uint16_t* xp, cudaStream_t s) {
  if (Tk == 0) return MOE_OK;
  note_launch();
  return check_cuda(launch_pdl(gather_rows_kernel, dim3(Tk), dim3(128), 0, s, x, perm, k, H, xp), "gather_rows_kernel");
}

}  // namespace moe
