// Grouped W4A16 GEMM path of the MoE layer for large token batches (prefill) ("Every Expert
// Counts: ExactMoE for Memory-Efficient W4A16 Inference", Abstract: all selected experts run
// through fused grouped MoE kernels).
//
// Launch sequence: permute (group pairs by expert) -> gather rows -> tile plan -> gate/up GEMM
// with fused silu(g)*u -> down GEMM (fp32 rows per token-expert pair) -> router-weighted combine.
//
// Both GEMMs are one persistent tcgen05 kernel (sm_100a). A CTA tile is a PAIR of 128-row
// weight blocks (gate rows f..f+127 and the matching up rows, or two consecutive row blocks of
// W2) against up to 128 tokens of one expert:
//   D_0[128 x N] = W_blk0 . X^T,  D_1[128 x N] = W_blk1 . X^T   (N = tokens, multiple of 16)
// The weights are the A operand and live in TENSOR MEMORY: 8 dequantiser warps turn each 128 x
// 128 int4 tile (TMA-staged in shared memory) into bf16 rows (q * s) and write them with
// tcgen05.st. The token rows are the B operand, loaded by TMA with 128-byte swizzle; one token
// tile feeds both MMAs, which keeps the shared-memory traffic per MMA flop low. Accumulators
// are fp32 in tensor memory; 4 epilogue warps drain them with tcgen05.ld.
// Tile list: per expert, ceil(n_e / 128) token chunks x row-block pairs; MMA N is the chunk's
// token count rounded up to 16, so a ragged tail costs at most 15 padded tokens per expert.
// Tiles are claimed dynamically (atomic counter). Every wait is bounded.
// Split K for the down GEMM: when the down tiles would fill the SMs only about once (few token
// chunks, long K = I), each tile's K range is split in two halves that run as separate tiles and
// add their fp32 partial rows into the zeroed output rows (two terms: the sum does not depend on
// which half comes first). This fills the second round of SMs with half-length
// tiles instead of leaving most of them idle while a few full-length tiles finish.
#include <algorithm>
#include <type_traits>
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "tc.cuh"

namespace moe {
namespace dec {
extern unsigned long long* g_trace;   // diagnostics buffer (moe_debug_set_decode_trace)
}
namespace {

constexpr int kGStages = 3;
constexpr int kGThreads = 480;      // 15 warps
constexpr int kGIssuer1 = 14;       // second MMA-issuing warp (block 1 of the pair)
constexpr int kGEpi0 = 2;           // warps 2..5
constexpr int kGDq0 = 6;            // warps 6..13
constexpr int kTokTile = 128;
constexpr int kGTmemCols = 512;
constexpr int kGA = 0;              // 2 A buffers x (64 gate + 64 up) columns
constexpr int kGD0 = 256;           // D_0 columns 256..383
constexpr int kGD1 = 384;           // D_1 columns 384..511
constexpr uint32_t kBBoxBytes = kTokTile * 128;   // one 64-wide K box of 128 rows (16 KB)

enum { kModeGateUp = 0, kModeDown = 1 };

struct __align__(1024) GStage {
  uint8_t b[2][kBBoxBytes];     // token rows, K 0..63 and 64..127 of the group (SW128)
  uint8_t w[2][8192];           // int4 tiles of block 0 and block 1 (16 chunks of 8 rows each)
  uint16_t sc[2][128];          // their scales, in row order
};

// Stage of the bf16-weight variant: one 64-wide K slice of the token rows and of both weight
// blocks, all three as 128-byte-swizzled K-major tiles straight from TMA (MMA operands in place).
struct __align__(1024) GStageBf {
  uint8_t b[kBBoxBytes];        // token rows, K slice of 64 (SW128)
  uint8_t a[2][kBBoxBytes];     // weight rows of block 0 and block 1, same K slice (SW128)
};

template <bool kBf16>
struct GSmem {
  typename std::conditional<kBf16, GStageBf, GStage>::type st[kGStages];
  uint16_t ostage[128][256];    // epilogue: the tile's outputs, token-major (bf16, 64 KB)
  uint64_t full[kGStages], empty[kGStages];
  uint64_t afull[2], aempty[2];
  uint64_t dfull, dempty;
  uint64_t tq_full[4], tq_empty[4];
  uint64_t drain[2];
  int tq[4];
  uint32_t tmem_base;
  int abort;
};

struct GParams {
  int rg_slot;                              // 8-row groups per slot (N / 8) of the matrix
  int K;                                    // H for gate/up, I for down
  int G;                                    // K / 128
  int rows_half;                            // gate/up: I (up block offset); down: unused
  int mode;
  int ksplit;                               // down: K halves per tile (1 or 2); gate/up: 1
  const int32_t* tile_list;                 // packed tiles
  const int32_t* ntiles;                    // total tile count (device)
  const int32_t* offsets;                   // grouped pair offsets [E+1]
  const int32_t* table;                     // expert -> slot (nullable)
  unsigned long long* trace;                // optional per-CTA clock stamps (diagnostics)
  const int32_t* perm;                      // pair id of grouped position
  const float* wts;                         // router weights [T*k] (applied by the combine)
  uint16_t* out;                            // gate/up: Hp [Tk][I] (bf16)
  float* y32;                               // down: Yp [Tk][H] (fp32, unweighted)
  int out_ld;                               // row length of out
  int Tk;
  int* ctl;
};

// packed tile: expert (8 bits) | chunk (12 bits) | block pair (12 bits)
__device__ __forceinline__ void unpack_tile(int32_t v, int& e, int& chunk, int& bp) {
  e = (v >> 24) & 0xff;
  chunk = (v >> 12) & 0xfff;
  bp = v & 0xfff;
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
      ::"r"(tc::smem_u32(dst)), "l"(map), "r"(x), "r"(y), "r"(tc::smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tma_load_2d_hint(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar,
                                                 uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;"
      ::"r"(tc::smem_u32(dst)), "l"(map), "r"(x), "r"(y), "r"(tc::smem_u32(bar)), "l"(policy)
      : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
        "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]),
        "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
        "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr)
      : "memory");
}

// diagnostics: 7 reference (after set-up); first tile of the CTA, K group g < 16:
// 48+g stage issued, 16+g dequantised A ready (warp 6), 32+g issuer 0 done issuing;
// 1 epilogue saw D of tile 0, 2 epilogue released D of tile 0, 3 issuer 0 starts tile 1
__device__ __forceinline__ void gtrace(const GParams& P, int slot) {
  if (P.trace) P.trace[blockIdx.x * 64 + slot] = (unsigned long long)clock64();
}

// Named barrier over `n` threads that also ANDs a flag over them (uniform decisions).
__device__ __forceinline__ bool bar_and(int id, int n, bool v) {
  uint32_t r;
  asm volatile("{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.and.pred q, %2, %3, p;\n\t"
               "selp.u32 %0, 1, 0, q;\n\t}"
               : "=r"(r) : "r"((uint32_t)v), "r"(id), "r"(n) : "memory");
  return r != 0;
}

__device__ __forceinline__ bool gwait(uint64_t* bar, uint32_t parity, volatile int* abort) {
  const bool ok = tc::mbar_wait(bar, parity, abort);
  return __all_sync(0xffffffffu, ok);
}

// Token-row maps of one operand with boxes of 128, 64 and 32 rows: a tile of at most 64 (32)
// tokens loads only those rows, so its stages carry fewer bytes and turn over faster. Then the
// weight bank's tile maps (codes, scales; see make_chunk_code_map).
struct alignas(64) BMaps {
  CUtensorMap m[3];
  CUtensorMap wc, ws;
};

struct TileDesc {
  int e, slot, chunk, bp, p0, ntok;
  int g0, g1;          // K groups [g0, g1) of this tile
  int part;            // K half (index of the partial output)
  size_t rb0, rb1;     // weight row blocks
};

// K range of a tile: the whole K, or one of two halves when K is split (the block-pair field
// then holds pair * 2 + half)
__device__ __forceinline__ void k_range(const GParams& P, int& bp, int& g0, int& g1, int& part) {
  if (P.ksplit == 2) {
    part = bp & 1;
    bp >>= 1;
    g0 = part ? P.G / 2 : 0;
    g1 = part ? P.G : P.G / 2;
  } else {
    part = 0;
    g0 = 0;
    g1 = P.G;
  }
}

__device__ __forceinline__ TileDesc describe(const GParams& P, int32_t packed) {
  TileDesc d;
  unpack_tile(packed, d.e, d.chunk, d.bp);
  k_range(P, d.bp, d.g0, d.g1, d.part);
  d.slot = slot_of(P.table, d.e);
  const int n_e = P.offsets[d.e + 1] - P.offsets[d.e];
  d.p0 = P.offsets[d.e] + d.chunk * kTokTile;
  d.ntok = min(kTokTile, n_e - d.chunk * kTokTile);
  if (P.mode == kModeGateUp) {
    d.rb0 = d.bp;
    d.rb1 = P.rows_half / kRowBlock + d.bp;
  } else {
    d.rb0 = 2 * d.bp;
    d.rb1 = 2 * d.bp + 1;
  }
  return d;
}

// kBf16: the weights are unquantised bf16 rows (the BF16 comparison configuration); a 2-D tensor
// map brings each 128-row x 64-K slice of both blocks into shared memory in the MMA's operand
// layout, the two issuers run tcgen05.mma with both operands in shared memory, and the
// dequantiser warps stay idle. Tile scheduling, epilogue and combine are the W4 kernel's.
template <bool kBf16>
__global__ void __launch_bounds__(kGThreads, 1)
grouped_gemm_kernel(const __grid_constant__ GParams P, const __grid_constant__ BMaps xm) {
  extern __shared__ __align__(1024) uint8_t gsmem_raw[];
  // the dynamic shared window is only guaranteed 16-byte aligned: align the carve-out by hand
  GSmem<kBf16>& s =
      *reinterpret_cast<GSmem<kBf16>*>((reinterpret_cast<uintptr_t>(gsmem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (tid == 0) {
    for (int i = 0; i < kGStages; ++i) {
      tc::mbar_init(&s.full[i], 1);
      tc::mbar_init(&s.empty[i], kBf16 ? 2 : 8 + 2);   // (8 dequant warps +) the two issuers' commits
    }
    for (int i = 0; i < 2; ++i) { tc::mbar_init(&s.afull[i], 8); tc::mbar_init(&s.aempty[i], 2); }
    tc::mbar_init(&s.dfull, 2);
    tc::mbar_init(&s.dempty, 4);
    for (int i = 0; i < 4; ++i) { tc::mbar_init(&s.tq_full[i], 1); tc::mbar_init(&s.tq_empty[i], kBf16 ? 2 + 4 : 2 + 4 + 8); }
    tc::mbar_init(&s.drain[0], 1);
    tc::mbar_init(&s.drain[1], 1);
    s.abort = 0;
    tc::fence_barrier_init();
    for (int i = 0; i < 3; ++i) asm volatile("prefetch.tensormap [%0];" ::"l"(&xm.m[i]) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(&xm.wc) : "memory");
    if (!kBf16) asm volatile("prefetch.tensormap [%0];" ::"l"(&xm.ws) : "memory");
  }
  if (warp == 1) {
    tc::tmem_alloc<kGTmemCols>(&s.tmem_base);
    tc::tc_fence_before();
  }
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = s.tmem_base;
  volatile int* abort = &s.abort;
  const int total = *P.ntiles;
  if (tid == 0) gtrace(P, 7);

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    const uint64_t pol_w = tc::policy_evict_last();   // weights are reused across token chunks
    int it = 0;
    for (int n = 0;; ++n) {
      int t = 0;
      if (lane == 0) t = atomicAdd(P.ctl + kCtlClaim, 1);
      t = __shfl_sync(0xffffffffu, t, 0);
      const bool stop = t >= total || *abort;
      const int q = n & 3;
      if (!gwait(&s.tq_empty[q], ((n >> 2) & 1) ^ 1, abort)) {
        if (lane == 0) report_status(P.ctl, MOE_ERR_TIMEOUT, 21);
        break;
      }
      if (lane == 0) {
        s.tq[q] = stop ? -1 : P.tile_list[t];
        tc::mbar_arrive(&s.tq_full[q]);
      }
      if (stop) break;
      const TileDesc d = describe(P, P.tile_list[t]);
      const int bi = d.ntok <= 32 ? 2 : (d.ntok <= 64 ? 1 : 0);   // token rows loaded: 128 >> bi
      const CUtensorMap* xmap = &xm.m[bi];
      const uint32_t bbytes = kBBoxBytes >> bi;
      // the pair's two 128-row blocks: row-group coordinates in the bank's tile maps
      const int z0 = d.slot * P.rg_slot + (int)d.rb0 * (kRowBlock / kRowGroup);
      const int z1 = d.slot * P.rg_slot + (int)d.rb1 * (kRowBlock / kRowGroup);
      bool ok = true;
      if constexpr (kBf16) {
        // 64-wide K slices; weight rows of block b at (slot * N + 128 * rb) of the bank's map
        const int y0 = d.slot * P.rg_slot * kRowGroup + (int)d.rb0 * kRowBlock;
        const int y1 = d.slot * P.rg_slot * kRowGroup + (int)d.rb1 * kRowBlock;
        for (int ks = 2 * d.g0; ks < 2 * d.g1; ++ks, ++it) {
          const int st = it % kGStages;
          if (!gwait(&s.empty[st], ((it / kGStages) & 1) ^ 1, abort)) { ok = false; break; }
          if (lane == 0) {
            GStageBf& S = s.st[st];
            tc::mbar_arrive_expect_tx(&s.full[st], bbytes + 2 * kBBoxBytes);
            tma_load_2d(S.b, xmap, ks * 64, d.p0, &s.full[st]);
            tma_load_2d_hint(S.a[0], &xm.wc, ks * 64, y0, &s.full[st], pol_w);
            tma_load_2d_hint(S.a[1], &xm.wc, ks * 64, y1, &s.full[st], pol_w);
          }
        }
      } else {
      for (int g = d.g0; g < d.g1; ++g, ++it) {
        const int st = it % kGStages;
        if (!gwait(&s.empty[st], ((it / kGStages) & 1) ^ 1, abort)) { ok = false; break; }
        if (lane == 0) {
          GStage& S = s.st[st];
          tc::mbar_arrive_expect_tx(&s.full[st], 2 * bbytes + 2 * 8192 + 2 * 256);
          tma_load_2d(S.b[0], xmap, g * 128, d.p0, &s.full[st]);
          tma_load_2d(S.b[1], xmap, g * 128 + 64, d.p0, &s.full[st]);
          tc::tma_load_3d(S.w[0], &xm.wc, 0, g, z0, &s.full[st], pol_w);
          tc::tma_load_3d(S.w[1], &xm.wc, 0, g, z1, &s.full[st], pol_w);
          tc::tma_load_3d(S.sc[0], &xm.ws, 0, g, z0, &s.full[st], pol_w);
          tc::tma_load_3d(S.sc[1], &xm.ws, 0, g, z1, &s.full[st], pol_w);
          if (it < 16) gtrace(P, 48 + it);
        }
      }
      }
      if (!ok) {
        if (lane == 0) report_status(P.ctl, MOE_ERR_TIMEOUT, 22);
        if (lane == 0) s.abort = 1;
        break;
      }
    }
    if (lane == 0) {   // no copy may still be landing when the CTA leaves
      const int n = it < kGStages ? it : kGStages;
      for (int i = 0; i < n; ++i) {
        const int j = it - 1 - i;
        volatile int never = 0;
        tc::mbar_wait(&s.full[j % kGStages], (j / kGStages) & 1, &never);
      }
    }
  } else if (warp == 1 || warp == kGIssuer1) {
    // ---------------------------------------------------------------- MMA issuers
    // issuer `me` runs the MMAs of block `me` of the pair into accumulator D_me: one MMA
    // costs its issuing thread about as much as its tensor-pipe time at these N, so two
    // issuers keep the pipe fed
    const int me = warp == 1 ? 0 : 1;
    if (lane == 0) {
      int it = 0, a_it = 0;
      for (int n = 0;; ++n) {
        const int q = n & 3;
        if (!tc::mbar_wait(&s.tq_full[q], (n >> 2) & 1, abort)) { report_status(P.ctl, MOE_ERR_TIMEOUT, 23); break; }
        const int packed = s.tq[q];
        tc::mbar_arrive(&s.tq_empty[q]);
        if (packed < 0) break;
        const TileDesc d = describe(P, packed);
        const int nmma = (d.ntok + 15) & ~15;
        const uint32_t idesc = tc::idesc_bf16_f32(128, nmma);
        if (!tc::mbar_wait(&s.dempty, (n & 1) ^ 1, abort)) { report_status(P.ctl, MOE_ERR_TIMEOUT, 24); break; }
        tc::tc_fence_after();
        if (me == 0 && n == 1) gtrace(P, 3);
        bool ok = true;
        if constexpr (kBf16) {
          for (int ks = 2 * d.g0; ks < 2 * d.g1; ++ks, ++it) {
            const int st = it % kGStages;
            if (!tc::mbar_wait(&s.full[st], (it / kGStages) & 1, abort)) { ok = false; break; }
            tc::tc_fence_after();
            const uint32_t bbase = tc::smem_u32(s.st[st].b), abase = tc::smem_u32(s.st[st].a[me]);
            const uint32_t dacc = tmem + (me ? kGD1 : kGD0);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t adesc = tc::smem_desc(abase + kk * 32, 16, 1024, 2);
              const uint64_t bdesc = tc::smem_desc(bbase + kk * 32, 16, 1024, 2);
              tc::mma_ss(dacc, adesc, bdesc, idesc, (ks > 2 * d.g0 || kk > 0) ? 1u : 0u);
            }
            tc::mma_commit(&s.empty[st]);
          }
        } else {
        for (int g = d.g0; g < d.g1; ++g, ++it, ++a_it) {
          const int st = it % kGStages, ab = a_it & 1;
          if (!tc::mbar_wait(&s.full[st], (it / kGStages) & 1, abort) ||
              !tc::mbar_wait(&s.afull[ab], (a_it >> 1) & 1, abort)) {
            ok = false;
            break;
          }
          tc::tc_fence_after();
          const uint32_t bbase = tc::smem_u32(s.st[st].b[0]);
          const uint32_t a = tmem + kGA + ab * 128 + me * 64, dacc = tmem + (me ? kGD1 : kGD0);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t baddr = bbase + (kk >> 2) * kBBoxBytes + (kk & 3) * 32;
            const uint64_t bdesc = tc::smem_desc(baddr, 16, 1024, 2);
            tc::mma_ts(dacc, a + kk * 8, bdesc, idesc, (g > d.g0 || kk > 0) ? 1u : 0u);
          }
          tc::mma_commit(&s.aempty[ab]);
          tc::mma_commit(&s.empty[st]);
          if (me == 0 && a_it < 16) gtrace(P, 32 + a_it);
        }
        }
        if (!ok) {
          report_status(P.ctl, MOE_ERR_TIMEOUT, 25);
          s.abort = 1;
          break;
        }
        tc::mma_commit(&s.dfull);
      }
      tc::mma_commit(&s.drain[me]);
      volatile int never = 0;
      tc::mbar_wait(&s.drain[me], 0, &never);
    }
    __syncwarp();
  } else if (warp >= kGDq0 && warp < kGDq0 + 8) {
    // ---------------------------------------------------------------- dequantisers -> TMEM
    if constexpr (!kBf16) {
    const int quarter = warp & 3, blk = (warp - kGDq0) >> 2;     // block 0 or 1 of the pair
    const int r = quarter * 32 + lane;
    const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16) + kGA + blk * 64;
    const __nv_bfloat162 off136 = __floats2bfloat162_rn(136.f, 136.f);
    int it = 0, a_it = 0;
    for (int n = 0;; ++n) {
      const int q = n & 3;
      if (!gwait(&s.tq_full[q], (n >> 2) & 1, abort)) break;
      const int packed = s.tq[q];
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&s.tq_empty[q]);
      if (packed < 0) break;
      int bp = packed & 0xfff, g0, g1, part;
      k_range(P, bp, g0, g1, part);
      bool ok = true;
      for (int g = g0; g < g1; ++g, ++it, ++a_it) {
        const int st = it % kGStages, ab = a_it & 1;
        if (!gwait(&s.full[st], (it / kGStages) & 1, abort)) { ok = false; break; }
        const uint8_t* wsrc = s.st[st].w[blk];
        uint4 c[4];
#pragma unroll
        // tile in shared memory: 16 chunks of 512 bytes, one per 8-row group
        for (int kq = 0; kq < 4; ++kq)
          c[kq] = *reinterpret_cast<const uint4*>(wsrc + (r >> 3) * kChunkBytes + piece_offset(kq, r & 7));
        const uint32_t sbits = s.st[st].sc[blk][r];
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&s.empty[st]);
        const uint32_t s2u = sbits | (sbits << 16);
        const __nv_bfloat162 s2 = *reinterpret_cast<const __nv_bfloat162*>(&s2u);
        if (!gwait(&s.aempty[ab], ((a_it >> 1) & 1) ^ 1, abort)) { ok = false; break; }
        tc::tc_fence_after();
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t words[8] = {c[2 * h].x, c[2 * h].y, c[2 * h].z, c[2 * h].w,
                                     c[2 * h + 1].x, c[2 * h + 1].y, c[2 * h + 1].z, c[2 * h + 1].w};
          uint32_t v[32];
#pragma unroll
          for (int w = 0; w < 8; ++w)
#pragma unroll
            for (int p = 0; p < 4; ++p) {
              const uint32_t t = ((words[w] >> (4 * p)) & 0x000F000Fu) | 0x43004300u;
              const __nv_bfloat162 qv = __hsub2(*reinterpret_cast<const __nv_bfloat162*>(&t), off136);
              const __nv_bfloat162 wv = __hmul2(qv, s2);
              v[w * 4 + p] = *reinterpret_cast<const uint32_t*>(&wv);
            }
          tc::tmem_st32(trow + ab * 128 + h * 32, v);
        }
        tc::tmem_wait_st();
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&s.afull[ab]);
        if (warp == kGDq0 && lane == 0 && a_it < 16) gtrace(P, 16 + a_it);
      }
      if (!ok) break;
    }
    }
  } else {
    // ---------------------------------------------------------------- epilogue (warps 2..5)
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16);
    for (int n = 0;; ++n) {
      const int q = n & 3;
      // every exit is decided by all four epilogue warps together (they meet at named barriers)
      if (!bar_and(1, 128, gwait(&s.tq_full[q], (n >> 2) & 1, abort))) break;
      const int packed = s.tq[q];
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&s.tq_empty[q]);
      if (packed < 0) break;
      const TileDesc d = describe(P, packed);
      if (!bar_and(1, 128, gwait(&s.dfull, n & 1, abort))) break;
      tc::tc_fence_after();
      if (warp == kGEpi0 && lane == 0 && n == 0) gtrace(P, 1);
      // the whole tile: tensor memory -> registers, then gate/up: h to shared memory (token-major,
      // bf16) for 16-byte coalesced stores of whole rows below; down: fp32 rows straight to global
      // memory. The accumulators are released as soon as they are read, so the next tile's MMAs
      // overlap the stores
      const int etid = tid - kGEpi0 * 32;
      for (int c0 = 0; c0 < d.ntok; c0 += 32) {
        uint32_t v0[32], v1[32];
        tmem_ld32(trow + kGD0 + c0, v0);
        tmem_ld32(trow + kGD1 + c0, v1);
        tc::tmem_wait_ld();
        if (P.mode == kModeGateUp) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            // silu(g) * u with the hardware exp and reciprocal: h is rounded to bf16 (8 bits)
            // right after, far coarser than their few-ulp fp32 error
            const float g = __uint_as_float(v0[j]), u = __uint_as_float(v1[j]);
            s.ostage[c0 + j][r] = __bfloat16_as_ushort(__float2bfloat16_rn(__fdividef(g * u, 1.f + __expf(-g))));
          }
        } else {
          // fp32 rows straight from the registers: for each token the warp's 32 lanes (rows)
          // write 128 contiguous bytes of each of the two row blocks. With the K split both
          // halves add into the zeroed row: 0 + a + b = 0 + b + a exactly, whichever comes first.
          float* yp = P.y32 + (size_t)(d.p0 + c0) * P.out_ld + (size_t)d.rb0 * kRowBlock + r;
          if (P.ksplit == 2) {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (c0 + j < d.ntok) {
                atomicAdd(yp + (size_t)j * P.out_ld, __uint_as_float(v0[j]));
                atomicAdd(yp + (size_t)j * P.out_ld + kRowBlock, __uint_as_float(v1[j]));
              }
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (c0 + j < d.ntok) {
                yp[(size_t)j * P.out_ld] = __uint_as_float(v0[j]);
                yp[(size_t)j * P.out_ld + kRowBlock] = __uint_as_float(v1[j]);
              }
          }
        }
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&s.dempty);
      if (warp == kGEpi0 && lane == 0 && n == 0) gtrace(P, 2);
      tc::named_bar_sync(1, 128);               // the staged tile is complete
      if (P.mode == kModeGateUp) {
        // 128 columns = 16 pieces of 16 bytes per token row; a warp stores two rows per step
        const size_t col = (size_t)d.bp * kRowBlock + (etid & 15) * 8;
        for (int t0 = 0; t0 < d.ntok; t0 += 32) {
          uint4 v[4];
#pragma unroll
          for (int m = 0; m < 4; ++m) v[m] = *reinterpret_cast<const uint4*>(&s.ostage[t0 + (etid >> 4) + 8 * m][(etid & 15) * 8]);
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            const int t = t0 + (etid >> 4) + 8 * m;
            if (t < d.ntok) *reinterpret_cast<uint4*>(P.out + (size_t)(d.p0 + t) * P.out_ld + col) = v[m];
          }
        }
      }
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc<kGTmemCols>(tmem);
  }
  if (tid == 0) {
    __threadfence();
    if (atomicAdd(P.ctl + kCtlDone, 1) == (int)gridDim.x - 1) {
      __threadfence();
      P.ctl[kCtlClaim] = 0;
      P.ctl[kCtlDone] = 0;
      __threadfence();
    }
  }
}

// One block per expert: writes that expert's tiles (chunk-major, block pair minor) at its
// prefix offset in the list, and block 0 writes the total.
__global__ void __launch_bounds__(256) tile_list_kernel(const int32_t* __restrict__ counts, int E,
                                                        const int32_t* __restrict__ table, int pairs,
                                                        int32_t* __restrict__ list, int32_t* __restrict__ total) {
  pdl_begin();
  const int e = blockIdx.x;
  __shared__ int base, mine;
  if (threadIdx.x == 0) {
    int b = 0, tot = 0;
    for (int x = 0; x < E; ++x) {
      const int n = (slot_of(table, x) >= 0) ? (counts[x] + kTokTile - 1) / kTokTile * pairs : 0;
      if (x < e) b += n;
      if (x == e) mine = n;
      tot += n;
    }
    base = b;
    if (e == 0) *total = tot;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < mine; i += blockDim.x) {
    const int chunk = i / pairs, bp = i % pairs;
    list[base + i] = (e << 24) | (chunk << 12) | bp;
  }
}

// out[t] = bf16( acc + sum_j wts[t][j] * y[inv[t][j]] ) over the fp32 down-projection rows y, in
// fixed j order.
__global__ void __launch_bounds__(256) combine_kernel(const float* __restrict__ yp, const float* __restrict__ wts,
                                                      const int32_t* __restrict__ idx,
                                                      const int32_t* __restrict__ inv,
                                                      const int32_t* __restrict__ table, int H, int k,
                                                      float* __restrict__ acc, bool accumulate,
                                                      uint16_t* __restrict__ out) {
  pdl_begin();
  const int t = blockIdx.x;
  const int n0 = (blockIdx.y * blockDim.x + threadIdx.x) * 8;
  if (n0 >= H) return;
  float v[8];
  float* accp = acc + (size_t)t * H + n0;
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = accumulate ? accp[i] : 0.f;
  for (int j = 0; j < k; ++j) {
    if (slot_of(table, idx[(size_t)t * k + j]) < 0) continue;
    const float w = wts[(size_t)t * k + j];
    const float* yrow = yp + (size_t)inv[(size_t)t * k + j] * H + n0;
    const float4 a0 = *reinterpret_cast<const float4*>(yrow), a1 = *reinterpret_cast<const float4*>(yrow + 4);
    const float yf[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = fmaf(w, yf[i], v[i]);
  }
  if (out) {
    uint32_t pk[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __nv_bfloat162 b = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
      pk[i] = *reinterpret_cast<const uint32_t*>(&b);
    }
    *reinterpret_cast<uint4*>(out + (size_t)t * H + n0) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    if (accumulate)
#pragma unroll
      for (int i = 0; i < 8; ++i) accp[i] = 0.f;
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) accp[i] = v[i];
  }
}

// ---------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

int get_encode() {
  if (g_encode) return MOE_OK;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
  if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn)
    return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return MOE_OK;
}

// 2-D map over a row-major bf16 matrix [rows][cols]: box = 64 columns x box_rows rows, 128B swizzle.
int make_rows_map(CUtensorMap* map, const void* base, int rows, int cols, int box_rows) {
  if (int rc = get_encode()) return rc;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return MOE_OK;
}

int g_sms = 0;
int sm_count() {
  if (!g_sms) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&g_sms, cudaDevAttrMultiProcessorCount, dev);
    if (g_sms <= 0) g_sms = 148;
  }
  return g_sms;
}

template <bool kBf16>
int launch_gemm(const GParams& P, const BMaps& map, int max_tiles, cudaStream_t s) {
  const size_t smem = sizeof(GSmem<kBf16>) + 1024;
  static bool attr = false;
  if (!attr) {
    if (int rc = check_cuda(cudaFuncSetAttribute(grouped_gemm_kernel<kBf16>,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem),
                            "grouped GEMM: smem attribute"))
      return rc;
    attr = true;
  }
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(std::max(1, std::min(sm_count(), max_tiles)));
  cfg.blockDim = dim3(kGThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attrs[1];
  attrs[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, grouped_gemm_kernel<kBf16>, P, map);
  note_launch();
  return check_cuda(e, "grouped_gemm_kernel launch");
}

}  // namespace

bool ffn_grouped_supported(const FfnArgs& a) {
  return a.T >= 1 && a.E <= kMaxExperts && a.H % 256 == 0 && a.I % kRowBlock == 0 && (size_t)a.T * a.k < (1u << 20) &&
         a.H / kRowBlock < 4096 && a.I / kRowBlock < 4096 &&   // 12-bit block field of a packed tile
         (a.T * a.k + kTokTile - 1) / kTokTile < 4096;
}

int ffn_grouped(const FfnArgs& a, cudaStream_t s) {
  const WsLayout L = ws_layout(a.T, a.H, a.I, a.E, a.k);
  const int Tk = a.T * a.k;
  int32_t* counts = reinterpret_cast<int32_t*>(a.ws + L.counts);
  int32_t* offsets = reinterpret_cast<int32_t*>(a.ws + L.offsets);
  int32_t* perm = reinterpret_cast<int32_t*>(a.ws + L.perm);
  int32_t* inv = reinterpret_cast<int32_t*>(a.ws + L.inv);
  int32_t* tiles = reinterpret_cast<int32_t*>(a.ws + L.tiles);      // [0]: gate/up total, [1]: down total
  int32_t* list_gu = reinterpret_cast<int32_t*>(a.ws + L.tile_list);
  int32_t* list_dn = list_gu + L.tile_list_len;
  uint16_t* xp = reinterpret_cast<uint16_t*>(a.ws + L.xp);
  uint16_t* hp = reinterpret_cast<uint16_t*>(a.ws + L.hp);
  int* ctl = reinterpret_cast<int*>(a.ws + L.status);

  if (int rc = launch_permute(a.idx, a.T, a.k, a.E, counts, offsets, perm, inv,
                              reinterpret_cast<int32_t*>(a.ws + L.perm_scratch), s))
    return rc;
  if (int rc = launch_gather_rows(a.x, perm, Tk, a.k, a.H, xp, s)) return rc;
  const int IB = a.I / kRowBlock, HP = a.H / 256;
  // K split of the down GEMM: two halves when even the fewest token chunks this batch can have
  // give fewer than two rounds of down tiles on the SMs, and K holds at least two groups
  const int min_chunks = (Tk + kTokTile - 1) / kTokTile;
  const int ksplit = (a.I / kGroup >= 2 && (long long)min_chunks * HP < 2LL * sm_count()) ? 2 : 1;
  note_launch();
  if (int rc = check_cuda(launch_pdl(tile_list_kernel, dim3(a.E), dim3(256), 0, s, (const int32_t*)counts, a.E, a.slot,
                                     IB, list_gu, tiles + 0), "tile_list_kernel"))
    return rc;
  note_launch();
  if (int rc = check_cuda(launch_pdl(tile_list_kernel, dim3(a.E), dim3(256), 0, s, (const int32_t*)counts, a.E, a.slot,
                                     HP * ksplit, list_dn, tiles + 1), "tile_list_kernel"))
    return rc;
  const int max_chunks = (Tk + kTokTile - 1) / kTokTile + a.E;

  BMaps xmap, hmap;
  for (int i = 0; i < 3; ++i) {
    if (int rc = make_rows_map(&xmap.m[i], xp, Tk, a.H, kTokTile >> i)) return rc;
    if (int rc = make_rows_map(&hmap.m[i], hp, Tk, a.I, kTokTile >> i)) return rc;
  }

  // the banks hold at least E slots' worth of addressable rows (slot indices are < E)
  if (a.bf16_weights) {
    // unquantised rows: [E * 2I][H] and [E * H][I] bf16, boxes of 128 rows x 64 K (128-byte swizzle)
    if (int rc = make_rows_map(&xmap.wc, a.w13, a.E * 2 * a.I, a.H, kRowBlock)) return rc;
    if (int rc = make_rows_map(&hmap.wc, a.w2, a.E * a.H, a.I, kRowBlock)) return rc;
  } else {
    if (int rc = make_chunk_code_map(&xmap.wc, a.w13, 2 * a.I, a.H, a.E)) return rc;
    if (int rc = make_chunk_scale_map(&xmap.ws, a.s13, 2 * a.I, a.H, a.E)) return rc;
    if (int rc = make_chunk_code_map(&hmap.wc, a.w2, a.H, a.I, a.E)) return rc;
    if (int rc = make_chunk_scale_map(&hmap.ws, a.s2, a.H, a.I, a.E)) return rc;
  }
  auto gemm = [&](const GParams& Pg, const BMaps& m, int max_tiles) {
    return a.bf16_weights ? launch_gemm<true>(Pg, m, max_tiles, s) : launch_gemm<false>(Pg, m, max_tiles, s);
  };

  GParams P{};
  P.rg_slot = 2 * a.I / kRowGroup;
  P.K = a.H; P.G = a.H / kGroup; P.rows_half = a.I; P.mode = kModeGateUp;
  P.ksplit = 1;
  P.tile_list = list_gu; P.ntiles = tiles + 0; P.offsets = offsets; P.table = a.slot;
  P.perm = perm; P.wts = a.wts; P.out = hp; P.out_ld = a.I; P.Tk = Tk; P.ctl = ctl;
  P.trace = nullptr;
  if (int rc = gemm(P, xmap, max_chunks * IB)) return rc;

  P.rg_slot = a.H / kRowGroup;
  P.K = a.I; P.G = a.I / kGroup; P.rows_half = 0; P.mode = kModeDown;
  // y per pair in fp32 (the one rounding left before the combine is the output's); with the K
  // split both halves add into rows zeroed first
  P.ksplit = ksplit;
  P.tile_list = list_dn; P.ntiles = tiles + 1; P.out = nullptr; P.out_ld = a.H;
  P.y32 = reinterpret_cast<float*>(a.ws + L.yp);                    // y per pair, fp32 [Tk][H]
  P.trace = dec::g_trace;
  if (ksplit == 2)
    if (int rc = check_cuda(cudaMemsetAsync(P.y32, 0, sizeof(float) * (size_t)Tk * a.H, s), "zero y")) return rc;
  if (int rc = gemm(P, hmap, max_chunks * HP * ksplit)) return rc;

  dim3 grid(a.T, ceil_div(a.H, 256 * 8));
  note_launch();
  return check_cuda(launch_pdl(combine_kernel, grid, dim3(256), 0, s, (const float*)P.y32, a.wts, a.idx,
                               (const int32_t*)inv, a.slot, a.H, a.k, reinterpret_cast<float*>(a.ws + L.acc),
                               a.accumulate, a.out),
                    "combine_kernel");
}

}  // namespace moe
