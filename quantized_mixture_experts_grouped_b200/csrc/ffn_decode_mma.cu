// Fused decode kernel for batches of at most sixteen tokens: routing, gate/up with SiLU*up, down
// projection and the router-weighted combine in ONE launch ("Every Expert Counts: ExactMoE for
// Memory-Efficient W4A16 Inference", Abstract: all selected experts execute through fused
// grouped MoE kernels; the router's top-k is unchanged).
//
// With at most sixteen tokens the layer is a skinny product over every selected expert's packed
// weights, bound by HBM bandwidth and by the latency of its dependent steps. The work split,
// partials and reductions are those of decode_common.cuh. The contraction runs on the warp-level
// integer tensor-core path (mma.sync m16n8k32, u8 x s8 -> s32), which takes the int4 codes
// almost as they are stored:
//  * weights: a packed word holds the codes c = q + 8 (0..15) of eight consecutive K elements,
//    element 2p at bits 4p and element 2p + 1 at bits 16 + 4p. w & 0x0F0F0F0F holds elements
//    (0, 4, 1, 5) and (w >> 4) & 0x0F0F0F0F elements (2, 6, 3, 7), one per byte: three logic
//    operations turn eight codes into eight u8 A-operand elements;
//  * activations (x in phase 1, h in phase 2): each 128-element group of one token is written as
//    the 16-bit fixed-point value v = rint(x / a), a = max|x| / 32639, split into two signed
//    bytes v = 256 hi + lo. hi and lo are two B-operand columns stored in the same permuted
//    element order, so one MMA covers 16 weight rows x 32 K elements for four tokens;
//  * 256 D_hi + D_lo - 8 sum(v) = sum_k q_k v_k is exact in s32, and times the row's bf16 scale
//    and the group's a it is the group's contribution in fp32. The one approximation is
//    |x - a v| <= a / 2 = max|x| / 65278 per element (bf16 rounding of a value near max|x| is up
//    to 128 times larger).
// The B columns of a tile are its expert's compact token list (the tokens routed to it), four
// tokens per MMA block, so an expert with n tokens costs ceil(n / 4) blocks, not T / 4. A compute
// warp does all 128 K of 16 rows of half the tiles of a stage (four MMAs into one accumulator per
// block), and the phase-2 h operands are copied into the activation area once phase 1 is over,
// so the ring's stages hold only codes and scales.
#include "decode_common.cuh"

namespace moe {
namespace dec {
namespace {

constexpr int kMWarps = 19;                // warp 0 producer, warps 1..16 compute, 17..18 epilogue
constexpr int kMThreads = kMWarps * 32;
constexpr int kMComputeWarps = 16;
constexpr int kMEpiWarp = 17;
constexpr int kMMaxStages = 6;
constexpr int kColPad = 64;                // bytes after each operand column: hi and lo columns of a token in
                                           // opposite bank halves (conflict-free 16-byte B loads)
constexpr int kHCol = kRowBlock + kColPad; // bytes per h column in a tile (128 K + pad)
constexpr int kRedStride = kRowBlock + 8;  // floats per (warp half, token) row of the block sums
// h bytes per (expert, K group) with KCOLS B columns: the columns, then one 16-byte record per
// token (two columns per token)
template <int KCOLS>
__host__ __device__ constexpr int kHTileOf() { return KCOLS * kHCol + KCOLS / 2 * 16; }

template <int TT>
struct Cfg {
  static constexpr int NB = (TT + 3) / 4;                 // MMAs per k-step (four tokens each)
  static constexpr int TC = TT < 4 ? TT : 4;              // tokens per epilogue chunk
  static constexpr int kCols = 8 * NB;                    // B columns (hi, lo per token)
  static constexpr int kHTile = kHTileOf<kCols>();         // h bytes per (expert, K group)
  static constexpr int kStageH = kTilesPerStage * kHTile;
  static constexpr int kStageBytes = kStageW + kStageS;    // one ring slot: codes and scales
};

template <int TT>
struct __align__(128) MSmem {
  uint64_t full[kMMaxStages], empty[kMMaxStages], hfull[kMMaxStages];
  RouteSmem rs;
  uint64_t redfull[2], redempty[2];
  float red[2][2][TT][kRedStride];     // block sums [buffer][warp half][token][row] (two buffers)
  int abort;
  // followed in dynamic shared memory by the activation area (phase 1: the columns
  // [kCols][H + kColPad] bytes and their group records [H/128][4 NB] x 16 B; phase 2: the ring
  // slots' h operands) and the stage ring (codes and scales)
};

// Compute warp cw works on rows r0 = 16 (cw % 8) + g and r0 + 8, all 128 K, of the tiles
// half, half + 2, ... of each stage (half = cw / 8); lane (g, c). These offsets are fixed for the
// warp.
struct LaneTile {
  int wofs;   // the lane's A words of K quarters 0, 1 in a tile (quarters 2, 3 follow 256 bytes on;
              // rows r0 and r0 + 8 are adjacent chunks)
  int woff;   // the lane's B words in a K group's column (16 bytes; the second half 64 bytes on)
  int r0, half;
};

// The B columns of the MMA blocks of one selected expert: its compact token list (RouteSmem::tok),
// four tokens (hi and lo columns) per block. boff[nb]: byte offset of the column that lane (g, c)
// reads in block nb; bm[nb] is all ones where that column holds a token and zero where not (the
// offset then points at a valid column and the mask clears what was read). roff[nb] / rm[nb]: the
// same for the record of the token whose sums the lane holds (compact token 4 nb + c).
template <int NB>
struct ColSet {
  int boff[NB], roff[NB];
  uint32_t bm[NB], rm[NB];
};

// This warp's tiles among tiles i0..i1-1 of a stage, NBA MMA blocks (compile time) of the expert's
// tokens, the loads of two tiles issued before their MMAs (one with more than four tokens). Phase 1: tile i is K group
// gi0 + i - i0 (mod nH) of the x columns xq (column stride fixed in boff) with the records at
// xrec + K group * rstride; phase 2: tile i's h operand is hq + i * kHTile, its records after the
// columns. Per block nb the four MMAs of the K group run into one accumulator (exact in s32); the
// tile's contribution is added to seg[nb][0 / 1] (compact token 4 nb + c, rows r0 / r0 + 8).
template <int PH, int NBA, int NB, int KCOLS>
__device__ __forceinline__ void run_tiles(const uint8_t* sw, const uint16_t* ss, const uint8_t* xq, const uint8_t* xrec,
                                          int rstride, int gi0, int nH, const uint8_t* hq, int i0, int i1,
                                          const LaneTile& L, const ColSet<NB>& cs, float (&seg)[NB][2]) {
  constexpr int KD = NBA == 1 ? 2 : 1;   // tiles whose loads go out together (registers permitting)
  const uint32_t M = 0x0F0F0F0Fu;
  for (int i = i0 + L.half; i < i1; i += 2 * KD) {
    uint2 w[KD][4];   // [tile][row r0 quarters 0-1, row r0 + 8 quarters 0-1, the same for quarters 2-3]
    float s0[KD], s1[KD];
    uint4 bx[KD][NBA][2];
    int4 rc[KD][NBA];
#pragma unroll
    for (int d = 0; d < KD; ++d) {
      const int ti = min(i + 2 * d, i1 - 1);   // past the end: reload the last tile, result unused
      const uint8_t* tb = sw + ti * kTileBytes + L.wofs;
      w[d][0] = *reinterpret_cast<const uint2*>(tb);
      w[d][1] = *reinterpret_cast<const uint2*>(tb + kChunkBytes);
      w[d][2] = *reinterpret_cast<const uint2*>(tb + 256);
      w[d][3] = *reinterpret_cast<const uint2*>(tb + kChunkBytes + 256);
      s0[d] = __uint_as_float((uint32_t)ss[ti * kRowBlock + L.r0] << 16);
      s1[d] = __uint_as_float((uint32_t)ss[ti * kRowBlock + L.r0 + 8] << 16);
      const uint8_t* bq;
      const uint8_t* rq;
      if constexpr (PH == 1) {
        int gd = gi0 + (ti - i0);
        while (gd >= nH) gd -= nH;
        bq = xq + gd * kGroup;
        rq = xrec + gd * rstride;
      } else {
        bq = hq + ti * kHTileOf<KCOLS>();
        rq = bq + KCOLS * kHCol;
      }
#pragma unroll
      for (int nb = 0; nb < NBA; ++nb) {
        const uint8_t* bp = bq + cs.boff[nb] + L.woff;
        uint4 v0 = *reinterpret_cast<const uint4*>(bp);
        uint4 v1 = *reinterpret_cast<const uint4*>(bp + 64);
        v0.x &= cs.bm[nb]; v0.y &= cs.bm[nb]; v0.z &= cs.bm[nb]; v0.w &= cs.bm[nb];
        v1.x &= cs.bm[nb]; v1.y &= cs.bm[nb]; v1.z &= cs.bm[nb]; v1.w &= cs.bm[nb];
        bx[d][nb][0] = v0;
        bx[d][nb][1] = v1;
        int4 r = *reinterpret_cast<const int4*>(rq + cs.roff[nb]);
        r.x &= (int)cs.rm[nb]; r.y &= (int)cs.rm[nb]; r.z &= (int)cs.rm[nb];
        rc[d][nb] = r;
      }
    }
#pragma unroll
    for (int d = 0; d < KD; ++d) {
      if (i + 2 * d >= i1) break;
#pragma unroll
      for (int nb = 0; nb < NBA; ++nb) {
        int acc[4] = {0, 0, 0, 0};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint2 wa = w[d][2 * h], wb = w[d][2 * h + 1];
          imma(acc, wa.x & M, wb.x & M, (wa.x >> 4) & M, (wb.x >> 4) & M, bx[d][nb][h].x, bx[d][nb][h].y);
          imma(acc, wa.y & M, wb.y & M, (wa.y >> 4) & M, (wb.y >> 4) & M, bx[d][nb][h].z, bx[d][nb][h].w);
        }
        const float a = __int_as_float(rc[d][nb].y);
        const int corr = rc[d][nb].x + rc[d][nb].z;
        const int v0 = acc[0] * 256 + acc[1] - corr;
        const int v1 = acc[2] * 256 + acc[3] - corr;
        seg[nb][0] = fmaf(s0[d] * a, (float)v0, seg[nb][0]);
        seg[nb][1] = fmaf(s1[d] * a, (float)v1, seg[nb][1]);
      }
    }
  }
}

// sum over c = c0..c1 (in that order) of partial entry (base + c), rows q*32 + lane of each
// quarter q, tokens t0 + i (i < TC, t0 + i < T): the loads of up to KB entries are issued before
// any is summed.
template <int TC, int KB>
__device__ __forceinline__ void sum_partials(const float* P0, int base, int c0, int c1, int T, int t0, int lane,
                                             float (&acc)[4][TC]) {
  for (int cb = c0; cb <= c1; cb += KB) {
    float v[KB][4][TC];
#pragma unroll
    for (int e = 0; e < KB; ++e) {
      const float* pp = P0 + (size_t)(base + cb + e) * T * kRowBlock + lane;
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int i = 0; i < TC; ++i)
          v[e][q][i] = (cb + e <= c1 && t0 + i < T) ? __ldcg(pp + (t0 + i) * kRowBlock + q * 32) : 0.f;
    }
#pragma unroll
    for (int e = 0; e < KB; ++e)
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int i = 0; i < TC; ++i) acc[q][i] += v[e][q][i];
  }
}

// The same for two ranges at once (gate and up partials of a feature block), entries t0 + i < nt
// of each partial (row stride T): each round issues the loads of up to KB entries of both before
// summing, each range in its own order.
template <int TC, int KB>
__device__ __forceinline__ void sum_partials2(const float* P0, int ba, int a0, int a1, float (&acc_a)[4][TC], int bb,
                                              int b0, int b1, float (&acc_b)[4][TC], int T, int nt, int t0, int lane) {
  for (int r = 0; a0 + r * KB <= a1 || b0 + r * KB <= b1; ++r) {
    float va[KB][4][TC], vb[KB][4][TC];
#pragma unroll
    for (int e = 0; e < KB; ++e) {
      const int ca = a0 + r * KB + e, cb = b0 + r * KB + e;
      const float* pa = P0 + (size_t)(ba + ca) * T * kRowBlock + lane;
      const float* pb = P0 + (size_t)(bb + cb) * T * kRowBlock + lane;
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int i = 0; i < TC; ++i) {
          const bool tok = t0 + i < nt;
          va[e][q][i] = (ca <= a1 && tok) ? __ldcg(pa + (t0 + i) * kRowBlock + q * 32) : 0.f;
          vb[e][q][i] = (cb <= b1 && tok) ? __ldcg(pb + (t0 + i) * kRowBlock + q * 32) : 0.f;
        }
    }
#pragma unroll
    for (int e = 0; e < KB; ++e)
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int i = 0; i < TC; ++i) {
          acc_a[q][i] += va[e][q][i];
          acc_b[q][i] += vb[e][q][i];
        }
  }
}

template <int TT>
__global__ void __launch_bounds__(kMThreads, 1) moe_decode_mma_kernel(const __grid_constant__ DecParams P,
                                                                      const __grid_constant__ DecMaps M) {
  using C = Cfg<TT>;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  MSmem<TT>& s = *reinterpret_cast<MSmem<TT>*>(smem_raw);
  const int xcs = P.H + kColPad;                                  // activation column stride (bytes)
  const int NS = P.nstages;
  // The activation area holds the x columns and their group records in phase 1, and the h
  // operands of the NS ring slots in phase 2 (copied there only once every CTA has finished
  // phase 1, when no x column is read any more). The stage ring follows it.
  uint8_t* xq = smem_raw + sizeof(MSmem<TT>);
  uint8_t* xrec = xq + (size_t)C::kCols * xcs;                    // [H/128][4 NB] group records
  const size_t xbytes = (size_t)C::kCols * xcs + (size_t)(P.H / kGroup) * 4 * C::NB * 16;
  const size_t xarea = xbytes > (size_t)NS * C::kStageH ? xbytes : (size_t)NS * C::kStageH;
  // the stage ring starts on a 128-byte boundary of the shared address space (tensor copies)
  uint8_t* ring_raw = xq + xarea;
  uint8_t* ring = ring_raw + (((tc::smem_u32(ring_raw) + 127u) & ~127u) - tc::smem_u32(ring_raw));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) trace_clk(P, 60);
  // ---- set-up that does not read the previous kernel's results: overlaps it under PDL
  if (warp == 0) {
    if (lane < kMMaxStages) {
      tc::mbar_init(&s.full[lane], 1);
      tc::mbar_init(&s.empty[lane], kMComputeWarps);
      tc::mbar_init(&s.hfull[lane], 1);
    }
    if (lane < 2) {
      tc::mbar_init(&s.redfull[lane], kMComputeWarps);
      tc::mbar_init(&s.redempty[lane], 1);
    }
    if (lane == 0) s.abort = 0;
    tc::fence_barrier_init();
  }
  route_clear(s.rs, tid, kMThreads);
  {
    // L2 prefetches of the logits and of this CTA's share of the activations' 128-byte lines (a
    // prefetch only warms L2, which stays coherent with the previous kernel's writes; the values
    // are read after the dependency wait), so that the later loads do not queue behind the weight
    // stream in HBM
    const int xl = (P.T * P.H * 2 + 127) / 128, ll = P.logits ? (P.T * P.E * 2 + 127) / 128 : 0;
    for (int i = blockIdx.x + gridDim.x * tid; i < xl; i += gridDim.x * kMThreads)
      asm volatile("prefetch.global.L2 [%0];" ::"l"(reinterpret_cast<const uint8_t*>(P.x) + (size_t)i * 128));
    if (blockIdx.x == 0)
      for (int i = tid; i < ll; i += kMThreads)
        asm volatile("prefetch.global.L2 [%0];" ::"l"(reinterpret_cast<const uint8_t*>(P.logits) + (size_t)i * 128));
  }
  __syncthreads();

  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (tid == 0) trace_at(P, 0);
  if (tid == 0) trace_clk(P, 61);
  route_begin(s.rs, P, tid, kMThreads);
  if (tid == 0) trace_clk(P, 62);
  __syncthreads();
  route_finish(s.rs, P, tid, kMThreads);
  if (tid == 0) { trace_at(P, 1); trace_clk(P, 7); }
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int G = gridDim.x, cta = blockIdx.x;
  Plan pl;
  pl.init(s.rs.nact, P.H, P.I, G, cta);
  // The activations of the tokens that this CTA's phase-1 experts take become B-operand columns
  // (x_encode, called by warps 1..18 while the producer's first copies are in flight): unit u is
  // (the u / nG-th such token, K group u % nG), warp w takes units w - 1, w + 17, ..., kXB units
  // per round whose loads (8 bytes per lane) are all issued before the first is encoded; a named
  // barrier among those warps ends it.
  auto x_encode = [&]() {
    constexpr int kXB = 8, kXWarps = kMWarps - 1;
    const int nG = P.H / kGroup;
    uint32_t need = 0;
    if (pl.e1 > pl.b1)
      for (int j = pl.b1 / pl.tpe1; j <= (pl.e1 - 1) / pl.tpe1; ++j)
        for (int i = 0; i < s.rs.ntok[j]; ++i) need |= 1u << s.rs.tok[j][i];
    const int xunits = __popc(need) * nG;
    auto token_of = [&](int u) {   // the (u / nG)-th token of the set
      uint32_t m = need;
      for (int r = u / nG; r > 0; --r) m &= m - 1;
      return __ffs(m) - 1;
    };
    uint2 xv[kXB];
    for (int u0 = warp - 1; u0 < xunits; u0 += kXB * kXWarps) {
#pragma unroll
      for (int r = 0; r < kXB; ++r) {
        const int u = u0 + r * kXWarps;
        if (u < xunits)
          xv[r] = *reinterpret_cast<const uint2*>(P.x + (size_t)token_of(u) * P.H + (u % nG) * kGroup + 4 * lane);
      }
#pragma unroll
      for (int r = 0; r < kXB; ++r) {
        const int u = u0 + r * kXWarps;
        if (u >= xunits) break;
        const float v[4] = {bf16_bits_to_float(xv[r].x & 0xffffu), bf16_bits_to_float(xv[r].x >> 16),
                            bf16_bits_to_float(xv[r].y & 0xffffu), bf16_bits_to_float(xv[r].y >> 16)};
        const int t = token_of(u), gq = u % nG, col = 8 * (t >> 2) + 2 * (t & 3);
        encode_group_c(v, xq + (size_t)col * xcs + gq * kGroup, xq + (size_t)(col + 1) * xcs + gq * kGroup,
                       reinterpret_cast<int4*>(xrec) + gq * 4 * C::NB + t, lane);
      }
    }
    tc::named_bar_sync(1, kXWarps * 32);
    if (tid == 32) trace_clk(P, 63);
  };
  volatile int* abort = &s.abort;
  const int T = P.T;
  const int rg13 = 2 * P.I / kRowGroup, rg2 = P.H / kRowGroup;   // 8-row groups per slot
  auto stage_w = [&](int st) { return ring + (size_t)st * C::kStageBytes; };
  auto stage_s = [&](int st) { return ring + (size_t)st * C::kStageBytes + kStageW; };
  auto stage_h = [&](int st) { return xq + (size_t)st * C::kStageH; };

  if (warp == 0) {
    // ------------------------------------------------------------ producer (whole warp)
    // lane 0 posts the expected bytes; lanes 0..2 issue the copies of a stage side by side
    const uint64_t pol = tc::policy_evict_first();
    int it = 0;
    bool ok = true, h_ready = false;
    int first2 = -1;
    int pend_n = 0, pend_st[kMMaxStages], pend_u[kMMaxStages], pend_len[kMMaxStages];
    int h_issued[kMMaxStages];
    for (int i = 0; i < kMMaxStages; ++i) h_issued[i] = 0;
    const int h_target = pl.m * pl.nI;
    auto issue_h = [&](int st, int u, int n) {
      const int j = (u % pl.tpr2) / pl.nI, g0 = u % pl.nI;
      if (lane == 0) tc::mbar_arrive_expect_tx(&s.hfull[st], (uint32_t)(n * C::kHTile));
      __syncwarp();
      if (lane == 2)
        tc::bulk_g2s(stage_h(st), P.hbuf + ((size_t)j * pl.nI + g0) * C::kHTile, (uint32_t)(n * C::kHTile),
                     &s.hfull[st], pol);
      ++h_issued[st];
    };
    auto wait_h = [&]() -> bool {
      int okw = 1;
      if (lane == 0) {
        const long long t0 = clock64();
        while (tc::ld_acquire(P.hdone) < h_target) {
          if (*abort || clock64() - t0 > tc::kWaitTimeoutCycles) {
            trace_val(P, 8, tc::ld_acquire(P.hdone));
            trace_val(P, 9, h_target);
            okw = 0;
            break;
          }
          __nanosleep(64);
        }
      }
      return __shfl_sync(kFull, okw, 0) != 0;
    };
    auto flush_h = [&]() -> bool {
      if (!h_ready) {
        if (!wait_h()) return false;
        fence_proxy_async_global();
        tc::fence_proxy_async_smem();   // the h copies overwrite the x columns read in phase 1
        h_ready = true;
        if (lane == 0) { trace_at(P, 4); trace_clk(P, 56); }
      }
      for (int i = 0; i < pend_n; ++i) issue_h(pend_st[i], pend_u[i], pend_len[i]);
      pend_n = 0;
      return true;
    };
    for (int phase = 1; phase <= 2 && ok; ++phase) {
      const int ub = phase == 1 ? pl.b1 : pl.b2, ue = phase == 1 ? pl.e1 : pl.e2;
      if (phase == 2 && ub < ue) first2 = it;
      for (int u = ub; u < ue; ++it) {
        const int n = phase == 1 ? pl.run1(u) : pl.run2(u);
        const int st = it % NS;
        // the slot about to be reused may hold a phase-2 stage still waiting for its h
        if (!h_ready && first2 >= 0 && it >= NS && it - NS >= first2 && !flush_h()) { ok = false; break; }
        if (!warp_wait(&s.empty[st], ((it / NS) & 1) ^ 1, abort)) { ok = false; break; }
        int j, lt;
        pl.locate(phase, u, j, lt);
        const int sl = s.rs.sl[j];
        if (lane == 0) tc::mbar_arrive_expect_tx(&s.full[st], (uint32_t)(n * (kTileBytes + kRowBlock * 2)));
        __syncwarp();
        // tile i of the stage: local tile lt + i = (row block, K group) of the expert's matrix;
        // lanes 0..3 load the codes, lanes 4..7 the scales, one tile each
        if (lane < 2 * kTilesPerStage && (lane & 3) < n) {
          const int i = lane & 3, nG = phase == 1 ? pl.nH : pl.nI;
          const int t = lt + i, rb = t / nG, gq = t - rb * nG;
          const int z = sl * (phase == 1 ? rg13 : rg2) + rb * (kRowBlock / kRowGroup);
          if (lane < kTilesPerStage)
            tc::tma_load_3d(stage_w(st) + i * kTileBytes, phase == 1 ? &M.c13 : &M.c2, 0, gq, z, &s.full[st], pol);
          else
            tc::tma_load_3d(stage_s(st) + i * kRowBlock * 2, phase == 1 ? &M.s13 : &M.s2, 0, gq, z, &s.full[st], pol);
        }
        if (lane == 0 && it < 8) trace_clk(P, 48 + it);
        if (phase == 2) {
          // h is waited for only when a slot holding a pending stage is needed again (or at the
          // end): until every CTA has finished phase 1 no phase-2 stage can be computed anyway
          if (h_ready) {
            if (!flush_h()) { ok = false; ++it; break; }
            issue_h(st, u, n);
          } else {
            pend_st[pend_n] = st; pend_u[pend_n] = u; pend_len[pend_n] = n; ++pend_n;
          }
        }
        u += n;
      }
    }
    if (lane == 0) trace_at(P, 3);
    if (ok && pend_n > 0 && !flush_h()) ok = false;
    if (!ok && lane == 0) {
      s.abort = 1;
      report_status(P.ctl, MOE_ERR_TIMEOUT, kSiteHDone);
    }
    if (lane == 0) {   // no bulk copy may still be landing in shared memory when the CTA leaves
      volatile int never = 0;
      const int nw = it < NS ? it : NS;
      for (int i = 0; i < nw; ++i) {
        const int jst = it - 1 - i;
        tc::mbar_wait(&s.full[jst % NS], (jst / NS) & 1, &never);
      }
      for (int st = 0; st < NS; ++st)
        if (h_issued[st] > 0) tc::mbar_wait(&s.hfull[st], (h_issued[st] - 1) & 1, &never);
    }
    __syncwarp();
  } else if (warp <= kMComputeWarps) {
    // ------------------------------------------------------------ compute warps 1..16
    x_encode();
    // warp cw = warp - 1 owns rows 16 * (cw % 8) .. + 15 and K half cw / 8 of every tile. The B
    // columns of a tile are its expert's compact token list, so an expert with n tokens takes
    // ceil(n / 4) MMA blocks. Phase 1: at the end of a W13 row block the two half sums of each
    // (row, compact token) go to shared memory (two buffers) for the epilogue warp. Phase 2: an
    // output block's buffer is cleared when the block starts, each expert's sums are added at the
    // token they belong to, and the buffer is handed over when the block ends. The compute warps go
    // on with the next tiles meanwhile.
    const int cw = warp - 1, kh = cw >> 3, g = lane >> 2, c = lane & 3;   // kh: the warp's plane of the block sums
    const int r0 = (cw & 7) * 16 + g;
    float seg[C::NB][2];
#pragma unroll
    for (int nb = 0; nb < C::NB; ++nb) { seg[nb][0] = 0.f; seg[nb][1] = 0.f; }
    // Stage bookkeeping without divisions: slot and parity, the current run's remaining tiles
    // (runs never cross an expert's W13 block or an output block's expert: the stage split the
    // producer makes with Plan::run1 / run2), the end of the current block and the K group.
    int it = 0, nblk = 0, st = 0;
    uint32_t ph = 0, hphase = 0;
    bool ok = true;
    LaneTile L;
    L.r0 = r0;
    L.half = kh;
    L.wofs = (r0 >> 3) * kChunkBytes + piece_offset(c >> 1, r0 & 7) + (c & 1) * 8;
    L.woff = 16 * c;
    ColSet<C::NB> cols;
    int nbe = 0, ne = 0, jcur = -1;
    long long tw[2][3] = {{0, 0, 0}, {0, 0, 0}};   // diagnostics: cycles waiting for data, in tiles, for buffers
    // the compact token columns of selected expert j (phase 1: the x columns of its tokens;
    // phase 2: the h tile's own columns, compact token i at columns 2 i, 2 i + 1 of block i / 4)
    auto setup = [&](int phase, int j) {
      jcur = j;
      ne = s.rs.ntok[j];
      nbe = (ne + 3) >> 2;
#pragma unroll
      for (int nb = 0; nb < C::NB; ++nb) {
        const int ib = 4 * nb + (g >> 1), ir = 4 * nb + c;
        const bool vb = ib < ne, vr = ir < ne;
        if (phase == 1) {
          const int tb = vb ? s.rs.tok[j][ib] : 0;
          cols.boff[nb] = (8 * (tb >> 2) + 2 * (tb & 3) + (g & 1)) * xcs;
          cols.roff[nb] = (vr ? s.rs.tok[j][ir] : 0) * 16;
        } else {
          cols.boff[nb] = vb ? (8 * nb + g) * kHCol : 0;
          cols.roff[nb] = vr ? ir * 16 : 0;
        }
        cols.bm[nb] = vb ? 0xffffffffu : 0u;
        cols.rm[nb] = vr ? 0xffffffffu : 0u;
      }
    };
    // tiles [i0, i1) of the stage in slot st (one expert), dispatched on its number of MMA blocks;
    // gi0 is the K group of tile i0 (phase 1)
    auto tiles = [&](int phase, int st, int i0, int i1, int gi0) {
      const uint8_t* sw = stage_w(st);
      const uint16_t* ss = reinterpret_cast<const uint16_t*>(stage_s(st));
      const uint8_t* hq = stage_h(st);
      const int rstride = 4 * C::NB * 16;
#define MOE_RUN(PH, NBA) run_tiles<PH, NBA, C::NB, C::kCols>(sw, ss, xq, xrec, rstride, gi0, pl.nH, hq, i0, i1, L, cols, seg)
      if (phase == 1) {
        if (nbe <= 1) MOE_RUN(1, 1);
        else if constexpr (C::NB >= 2) {
          if (nbe == 2) MOE_RUN(1, (C::NB >= 2 ? 2 : 1));
          else if constexpr (C::NB >= 4) {
            if (nbe == 3) MOE_RUN(1, 3); else MOE_RUN(1, 4);
          }
        }
      } else {
        if (nbe <= 1) MOE_RUN(2, 1);
        else if constexpr (C::NB >= 2) {
          if (nbe == 2) MOE_RUN(2, (C::NB >= 2 ? 2 : 1));
          else if constexpr (C::NB >= 4) {
            if (nbe == 3) MOE_RUN(2, 3); else MOE_RUN(2, 4);
          }
        }
      }
#undef MOE_RUN
    };
    for (int phase = 1; phase <= 2 && ok; ++phase) {
      const int ub = phase == 1 ? pl.b1 : pl.b2, ue = phase == 1 ? pl.e1 : pl.e2;
      if (ub >= ue) continue;
      const int per = phase == 1 ? pl.nH : pl.tpr2;       // tiles per block
      const int runlen = phase == 1 ? pl.tpe1 : pl.nI;    // tiles per contiguous run
      int blk_end = min(ue, (ub / per + 1) * per);
      int run_left = runlen - ub % runlen;
      int gk = ub % pl.nH;                                // K group of the next tile (phase 1)
      bool blk_new = true;                                // phase 2: next stage starts a block
      jcur = -1;
      for (int u = ub; u < ue && ok; ++it) {
        const int n = min(kTilesPerStage, min(ue - u, run_left));
        int jst, lt;
        pl.locate(phase, u, jst, lt);
        if (jst != jcur) setup(phase, jst);
        if (phase == 2 && blk_new) {
          // claim the output block's buffer and clear this lane's entries of every token
          const int b = nblk & 1;
          if (nblk >= 2 && !warp_wait(&s.redempty[b], ((nblk >> 1) - 1) & 1, abort)) { ok = false; break; }
          if (c == 0)
            for (int t = 0; t < T; ++t) {
              s.red[b][kh][t][r0] = 0.f;
              s.red[b][kh][t][r0 + 8] = 0.f;
            }
          __syncwarp();
          blk_new = false;
        }
        long long tq = P.trace ? clock64() : 0;
        if (!warp_wait(&s.full[st], ph, abort)) { ok = false; break; }
        if (phase == 2) {
          if (!warp_wait(&s.hfull[st], (hphase >> st) & 1, abort)) { ok = false; break; }
          hphase ^= 1u << st;
        }
        if (P.trace) { const long long t1 = clock64(); tw[phase - 1][0] += t1 - tq; tq = t1; }
        if (lane == 0 && cw == 0 && it < 8) trace_clk(P, 16 + it);
        if (phase == 1) {
          // the stage's tiles in segments that end at W13 row-block ends
          for (int i0 = 0; i0 < n && ok;) {
            const int i1 = min(n, blk_end - u);
            tiles(1, st, i0, i1, gk + i0 < pl.nH ? gk + i0 : (gk + i0) % pl.nH);
            if (P.trace) { const long long t1 = clock64(); tw[0][1] += t1 - tq; tq = t1; }
            if (u + i1 == blk_end) {
              const int b = nblk & 1;
              if (nblk >= 2 && !warp_wait(&s.redempty[b], ((nblk >> 1) - 1) & 1, abort)) { ok = false; break; }
              if (P.trace) { const long long t1 = clock64(); tw[0][2] += t1 - tq; tq = t1; }
#pragma unroll
              for (int nb = 0; nb < C::NB; ++nb) {
                const int ic = 4 * nb + c;
                if (nb < nbe && ic < ne) {
                  s.red[b][kh][ic][r0] = seg[nb][0];
                  s.red[b][kh][ic][r0 + 8] = seg[nb][1];
                }
                seg[nb][0] = 0.f;
                seg[nb][1] = 0.f;
              }
              __syncwarp();
              if (lane == 0) tc::mbar_arrive(&s.redfull[b]);
              ++nblk;
              blk_end = min(ue, blk_end + per);
            }
            i0 = i1;
          }
        } else {
          tiles(2, st, 0, n, 0);
          if (P.trace) { const long long t1 = clock64(); tw[1][1] += t1 - tq; tq = t1; }
        }
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&s.empty[st]);
        if (lane == 0 && cw == 0 && it < 8) trace_clk(P, 24 + it);
        if (phase == 2 && ok && (run_left == n || u + n == blk_end)) {
          // the expert's sums are complete for this block: add them at their tokens
          const int b = nblk & 1;
#pragma unroll
          for (int nb = 0; nb < C::NB; ++nb) {
            const int ic = 4 * nb + c;
            if (nb < nbe && ic < ne) {
              const int t = s.rs.tok[jcur][ic];
              s.red[b][kh][t][r0] += seg[nb][0];
              s.red[b][kh][t][r0 + 8] += seg[nb][1];
            }
            seg[nb][0] = 0.f;
            seg[nb][1] = 0.f;
          }
          if (u + n == blk_end) {
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&s.redfull[b]);
            ++nblk;
            blk_end = min(ue, blk_end + per);
            blk_new = true;
          }
        }
        u += n;
        gk += n;
        while (gk >= pl.nH) gk -= pl.nH;
        run_left -= n;
        if (run_left == 0) run_left = runlen;
        if (++st == NS) { st = 0; ph ^= 1; }
      }
    }
    if (P.trace && lane == 0) {   // diagnostics: warp 1 (both phases) in slots 10..15, warp 16 (phase 1) in 57..59
      unsigned long long* tr = P.trace + blockIdx.x * 64;
      if (cw == 0)
        for (int q = 0; q < 6; ++q) tr[10 + q] = (unsigned long long)tw[q / 3][q % 3];
      if (cw == kMComputeWarps - 1)
        for (int q = 0; q < 3; ++q) tr[57 + q] = (unsigned long long)tw[0][q];
    }
  } else {
    // ------------------------------------------------------------ epilogue warps
    // epilogue warp ew takes the blocks written to block-sum buffer ew (every other block), so
    // the reductions of consecutive blocks run side by side: half sums -> this CTA's partial; the
    // arrival that completes a block does its reduction (h of a feature block, or an output row
    // block), tokens in chunks of C::TC.
    constexpr int TC = C::TC;
    x_encode();
    const int ew = warp - kMEpiWarp;
    int nblk = 0, nh = 0;
    for (int phase = 1; phase <= 2; ++phase) {
      const int ub = phase == 1 ? pl.b1 : pl.b2, ue = phase == 1 ? pl.e1 : pl.e2;
      if (ub >= ue) continue;
      const int per = phase == 1 ? pl.nH : pl.tpr2;
      bool stop = false;
      for (int key = ub / per; key <= (ue - 1) / per; ++key, ++nblk) {
        const int b = nblk & 1;
        if (b != ew) continue;
        if (!warp_wait(&s.redfull[b], (nblk >> 1) & 1, abort)) { stop = true; break; }
        // phase 1: the block's expert's compact tokens; phase 2: every token
        const int nrow = phase == 1 ? (int)s.rs.ntok[key / (2 * pl.nI)] : T;
        float* part = (phase == 1 ? P.p1 : P.p2) + (size_t)(key + cta) * T * kRowBlock;
        for (int t = 0; t < nrow; ++t)
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int row = q * 32 + lane;
            part[t * kRowBlock + row] = s.red[b][0][t][row] + s.red[b][1][t][row];
          }
        __syncwarp();   // the buffer is read and the lanes' stores are ordered before lane 0's release
        if (lane == 0) tc::mbar_arrive(&s.redempty[b]);
        int last = 0;
        if (lane == 0) last = block_arrive(pl, P, phase, key) ? 1 : 0;
        last = __shfl_sync(kFull, last, 0);
        if (nblk < 8 && lane == 0) trace_clk(P, 32 + nblk);
        if (!last) continue;
        if (phase == 1) {
          // h = w * silu(gate) * up for feature block fb of selected expert j, encoded as the B
          // operand of the down projection
          const int nI = pl.nI, j = key / (2 * nI), fb = (key % (2 * nI)) % nI;
          if (lane == 0 && nh < 4) trace_clk(P, 40 + 2 * nh);
          // compact token i of the expert: h column pair i (hi, lo) and record i of the tile
          float wt = 0.f;
          if (lane < nrow) wt = route_weight(s.rs, P, s.rs.tok[j][lane], s.rs.act[j]);
          uint8_t* ht = P.hbuf + ((size_t)j * nI + fb) * C::kHTile;
          const int Rg = j * 2 * nI + fb, Ru = Rg + nI;
          for (int t0 = 0; t0 < nrow; t0 += TC) {
            float gs[4][TC], us[4][TC];
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
              for (int i = 0; i < TC; ++i) { gs[q][i] = 0.f; us[q][i] = 0.f; }
            sum_partials2<TC, (TC == 1 ? 4 : 1)>(P.p1, Rg, pl.first1(Rg), pl.last1(Rg), gs, Ru, pl.first1(Ru),
                                                  pl.last1(Ru), us, T, nrow, t0, lane);
#pragma unroll
            for (int i = 0; i < TC; ++i) {
              const int t = t0 + i;
              if (t < nrow) {
                const float w = __shfl_sync(kFull, wt, t);
                float hv[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) hv[q] = (w != 0.f) ? swiglu(gs[q][i], us[q][i]) * w : 0.f;
                const int col = 8 * (t >> 2) + 2 * (t & 3);
                encode_group(hv, ht + col * kHCol, ht + (col + 1) * kHCol,
                             reinterpret_cast<int4*>(ht + C::kCols * kHCol) + t, lane);
              }
            }
          }
          fence_proxy_async_global();
          __syncwarp();   // the lanes' stores are ordered before lane 0's release
          if (lane == 0) tc::red_release_add(P.hdone, 1);
          if (lane == 0 && nh < 4) trace_clk(P, 41 + 2 * nh);
          ++nh;
        } else {
          // output row block `key`: rows q*32 + lane, partials in CTA order, then the combine
          for (int t0 = 0; t0 < T; t0 += TC) {
            float yo[4][TC];
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
              for (int i = 0; i < TC; ++i) yo[q][i] = 0.f;
            sum_partials<TC, (TC == 1 ? 12 : 8 / TC)>(P.p2, key, pl.first2(key), pl.last2(key), T, t0, lane, yo);
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
              for (int i = 0; i < TC; ++i)
                if (t0 + i < T) store_output(P, t0 + i, key * kRowBlock + q * 32 + lane, yo[q][i]);
          }
        }
      }
      if (stop) break;
    }
    if (lane == 0) trace_at(P, 5);
  }

  __syncthreads();
  finish_launch(pl, P, abort, tid, kMThreads);
}

// Shared memory of a launch with ns ring slots: the fixed part, the activation area (x columns
// and records, or the ns slots' h operands, whichever is larger) and the ring.
template <int TT>
size_t smem_total(int H, int ns) {
  using C = Cfg<TT>;
  const size_t x = (size_t)C::kCols * (H + kColPad) + (size_t)(H / kGroup) * 4 * C::NB * 16;
  return sizeof(MSmem<TT>) + std::max(x, (size_t)ns * C::kStageH) + 128 + (size_t)ns * C::kStageBytes;
}

template <int TT>
int stages_tt(int H) {
  for (int ns = kMMaxStages; ns >= 1; --ns)
    if (smem_total<TT>(H, ns) <= (size_t)kSmemLimit) return ns;
  return 0;
}

template <int TT>
int launch_tt(const DecParams& P0, const DecMaps& M, int grid, cudaStream_t s) {
  DecParams P = P0;
  P.nstages = stages_tt<TT>(P.H);
  const size_t smem = smem_total<TT>(P.H, P.nstages);
  static bool attr_done = false;
  if (!attr_done) {
    if (int rc = check_cuda(cudaFuncSetAttribute(moe_decode_mma_kernel<TT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 kSmemLimit), "fused decode (warp MMA): smem attribute"))
      return rc;
    attr_done = true;
  }
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kMThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, moe_decode_mma_kernel<TT>, P, M);
  note_launch();
  return check_cuda(e, "moe_decode_mma_kernel launch");
}

int tt_of(int T) { return T <= 1 ? 1 : (T <= 2 ? 2 : (T <= 4 ? 4 : (T <= 8 ? 8 : 16))); }

}  // namespace

size_t mma_hbuf_per_tile(int T) {
  switch (tt_of(T)) {
    case 1: return Cfg<1>::kHTile;
    case 2: return Cfg<2>::kHTile;
    case 4: return Cfg<4>::kHTile;
    case 8: return Cfg<8>::kHTile;
    default: return Cfg<16>::kHTile;
  }
}

int mma_stages(int T, int H) {
  switch (tt_of(T)) {
    case 1: return stages_tt<1>(H);
    case 2: return stages_tt<2>(H);
    case 4: return stages_tt<4>(H);
    case 8: return stages_tt<8>(H);
    default: return stages_tt<16>(H);
  }
}

int launch_decode_mma(const DecParams& P, int grid, cudaStream_t s) {
  DecMaps M;
  if (int rc = make_chunk_code_map(&M.c13, P.w13, 2 * P.I, P.H, P.E)) return rc;
  if (int rc = make_chunk_scale_map(&M.s13, P.s13, 2 * P.I, P.H, P.E)) return rc;
  if (int rc = make_chunk_code_map(&M.c2, P.w2, P.H, P.I, P.E)) return rc;
  if (int rc = make_chunk_scale_map(&M.s2, P.s2, P.H, P.I, P.E)) return rc;
  switch (tt_of(P.T)) {
    case 1: return launch_tt<1>(P, M, grid, s);
    case 2: return launch_tt<2>(P, M, grid, s);
    case 4: return launch_tt<4>(P, M, grid, s);
    case 8: return launch_tt<8>(P, M, grid, s);
    default: return launch_tt<16>(P, M, grid, s);
  }
}

}  // namespace dec
}  // namespace moe
