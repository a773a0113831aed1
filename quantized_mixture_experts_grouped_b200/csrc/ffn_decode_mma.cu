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
// One MMA consumes 512 weights; a 128 x 128 tile takes 32 of them (8 per SM sub-partition),
// against about 16 FP32 instructions per 32 weights on the CUDA cores.
#include "decode_common.cuh"

namespace moe {
namespace dec {
namespace {

constexpr int kMWarps = 19;                // warp 0 producer, warps 1..16 compute, 17..18 epilogue
constexpr int kMThreads = kMWarps * 32;
constexpr int kMComputeWarps = 16;
constexpr int kMEpiWarp = 17;
constexpr int kMMaxStages = 6;
constexpr int kColPad = 32;                // bytes after each operand column (bank spread)
constexpr int kHCol = kRowBlock + kColPad; // bytes per h column in a tile (128 K + pad)
constexpr int kRedStride = kRowBlock + 8;  // floats per (half, token) row of the block sums

template <int TT>
struct Cfg {
  static constexpr int NB = (TT + 3) / 4;                 // MMAs per k-step (four tokens each)
  static constexpr int TC = TT < 4 ? TT : 4;              // tokens per epilogue chunk
  static constexpr int kCols = 8 * NB;                    // B columns (hi, lo per token)
  static constexpr int kHTile = kCols * kHCol + 4 * NB * 16;   // h bytes per (expert, K group)
  static constexpr int kStageH = kTilesPerStage * kHTile;
  static constexpr int kStageBytes = kStageW + kStageS + kStageH;
};

template <int TT>
struct __align__(128) MSmem {
  uint64_t full[kMMaxStages], empty[kMMaxStages], hfull[kMMaxStages];
  RouteSmem rs;
  uint64_t redfull[2], redempty[2];
  float red[2][2][TT][kRedStride];     // per-half block sums (two buffers)
  int abort;
  // followed in dynamic shared memory by the activation columns [kCols][H + kColPad] (bytes),
  // their group records [H/128][4 NB] x 16 B and the stage ring
};

// One 128 x 128 tile for compute warp (mt, kh): rows mt*16 + g and + 8, K half kh, lane (g, c).
// tile_issue loads the operands and issues the MMAs; tile_finish adds the tile's contribution,
// so that the next tile's MMAs can be issued before this one's results are needed.
template <int NB>
struct TileAcc {
  int d[NB][4];             // accumulators (token 4 nb + c: hi, lo columns of rows r0, r0 + 8)
  float sa0[NB], sa1[NB];   // row scale x group scale a of token 4 nb + c (0 for tokens >= T)
  int corr[NB];             // 8 * sum(v) over the K half
};

// tb: the packed tile; sc: its 128 row scales; bcol: B column 0 at the tile's first word, column
// stride cs bytes; rec: the K group's records (16 B per token).
template <int NB>
__device__ __forceinline__ void tile_issue(const uint8_t* tb, const uint16_t* sc, const uint8_t* bcol, int cs,
                                           const uint8_t* rec, int r0, int kh, int g, int c, int T, TileAcc<NB>& A) {
  // the tile is 16 chunks of 512 bytes, one per 8-row group (rows r0 and r0 + 8: adjacent chunks)
  const int q = 2 * kh + (c >> 1);
  const uint8_t* p0 = tb + (r0 >> 3) * kChunkBytes + piece_offset(q, r0 & 7) + (c & 1) * 8;
  const uint2 w0 = *reinterpret_cast<const uint2*>(p0);
  const uint2 w1 = *reinterpret_cast<const uint2*>(p0 + kChunkBytes);
  const uint32_t M = 0x0F0F0F0Fu;
  const uint32_t a0 = w0.x & M, a1 = w1.x & M, a2 = (w0.x >> 4) & M, a3 = (w1.x >> 4) & M;
  const uint32_t b0 = w0.y & M, b1 = w1.y & M, b2 = (w0.y >> 4) & M, b3 = (w1.y >> 4) & M;
  const float s0 = __uint_as_float((uint32_t)sc[r0] << 16), s1 = __uint_as_float((uint32_t)sc[r0 + 8] << 16);
  const int woff = (8 * kh + 2 * c) * 8;   // this lane's two words of the K half
#pragma unroll
  for (int nb = 0; nb < NB; ++nb) {
    const int n = 8 * nb + g;
    uint4 bx = make_uint4(0u, 0u, 0u, 0u);
    if (n < 2 * T) bx = *reinterpret_cast<const uint4*>(bcol + n * cs + woff);
#pragma unroll
    for (int e = 0; e < 4; ++e) A.d[nb][e] = 0;
    imma(A.d[nb], a0, a1, a2, a3, bx.x, bx.y);
    imma(A.d[nb], b0, b1, b2, b3, bx.z, bx.w);
    const int t = 4 * nb + c;
    A.sa0[nb] = 0.f; A.sa1[nb] = 0.f; A.corr[nb] = 0;
    if (t < T) {
      const int2 rc = *reinterpret_cast<const int2*>(rec + t * 16 + kh * 8);
      const float a = __int_as_float(rc.y);
      A.sa0[nb] = s0 * a;
      A.sa1[nb] = s1 * a;
      A.corr[nb] = rc.x;
    }
  }
}

// seg[nb][0 / 1]: token 4 nb + c, rows r0 / r0 + 8.
template <int NB>
__device__ __forceinline__ void tile_finish(const TileAcc<NB>& A, float (&seg)[NB][2]) {
#pragma unroll
  for (int nb = 0; nb < NB; ++nb) {
    const int v0 = A.d[nb][0] * 256 + A.d[nb][1] - A.corr[nb];
    const int v1 = A.d[nb][2] * 256 + A.d[nb][3] - A.corr[nb];
    seg[nb][0] = fmaf(A.sa0[nb], (float)v0, seg[nb][0]);
    seg[nb][1] = fmaf(A.sa1[nb], (float)v1, seg[nb][1]);
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

// The same for two ranges at once (gate and up partials of a feature block): each round issues
// the loads of up to KB entries of both before summing, each range in its own order.
template <int TC, int KB>
__device__ __forceinline__ void sum_partials2(const float* P0, int ba, int a0, int a1, float (&acc_a)[4][TC], int bb,
                                              int b0, int b1, float (&acc_b)[4][TC], int T, int t0, int lane) {
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
          const bool tok = t0 + i < T;
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
  uint8_t* xq = smem_raw + sizeof(MSmem<TT>);
  uint8_t* xrec = xq + (size_t)C::kCols * xcs;                    // [H/128][4 NB] group records
  // the stage ring starts on a 128-byte boundary of the shared address space (tensor copies)
  uint8_t* ring_raw = xrec + (size_t)(P.H / kGroup) * 4 * C::NB * 16;
  uint8_t* ring = ring_raw + (((tc::smem_u32(ring_raw) + 127u) & ~127u) - tc::smem_u32(ring_raw));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int NS = P.nstages;

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
  __syncthreads();

  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (tid == 0) trace_at(P, 0);
  if (tid == 0) trace_clk(P, 61);
  // activations as B-operand columns: warp w encodes the (token, K group) units w, w + 19, ...;
  // the loads of its first unit are issued before the routing so the latencies overlap
  {
    const int nG = P.H / kGroup, units = nG * P.T;
    float v[4];
    auto load = [&](int u) {
      const uint16_t* xp = P.x + (size_t)(u / nG) * P.H + (u % nG) * kGroup + lane;
#pragma unroll
      for (int q = 0; q < 4; ++q) v[q] = bf16_bits_to_float(xp[q * 32]);
    };
    if (warp < units) load(warp);
    route_begin(s.rs, P, tid, kMThreads);
    if (tid == 0) trace_clk(P, 62);
    for (int u = warp; u < units; u += kMWarps) {
      if (u != warp) load(u);
      const int t = u / nG, G = u % nG, col = 8 * (t >> 2) + 2 * (t & 3);
      encode_group(v, xq + (size_t)col * xcs + G * kGroup, xq + (size_t)(col + 1) * xcs + G * kGroup,
                   reinterpret_cast<int4*>(xrec) + G * 4 * C::NB + t, lane);
    }
  }
  __syncthreads();
  if (tid == 0) trace_clk(P, 63);
  route_finish(s.rs, P, tid, kMThreads);
  if (tid == 0) { trace_at(P, 1); trace_clk(P, 7); }
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  const int G = gridDim.x, cta = blockIdx.x;
  Plan pl;
  pl.init(s.rs.nact, P.H, P.I, G, cta);
  volatile int* abort = &s.abort;
  const int T = P.T;
  const int rg13 = 2 * P.I / kRowGroup, rg2 = P.H / kRowGroup;   // 8-row groups per slot
  auto stage_w = [&](int st) { return ring + (size_t)st * C::kStageBytes; };
  auto stage_s = [&](int st) { return ring + (size_t)st * C::kStageBytes + kStageW; };
  auto stage_h = [&](int st) { return ring + (size_t)st * C::kStageBytes + kStageW + kStageS; };

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
    // warp cw = warp - 1 owns rows 16 * (cw % 8) .. + 15 and K half cw / 8 of every tile. At the
    // end of a block the two half sums of each (row, token) go to shared memory (two buffers) for
    // the epilogue warp; the compute warps go on with the next tiles.
    const int cw = warp - 1, kh = cw >> 3, g = lane >> 2, c = lane & 3;
    const int r0 = (cw & 7) * 16 + g;
    float seg[C::NB][2];
#pragma unroll
    for (int nb = 0; nb < C::NB; ++nb) { seg[nb][0] = 0.f; seg[nb][1] = 0.f; }
    // Stage bookkeeping without divisions: slot and parity, the current run's remaining tiles
    // (runs never cross an expert's W13 block or an output block's K groups: the stage split the
    // producer makes with Plan::run1 / run2), the end of the current block and the K group.
    int it = 0, nblk = 0, st = 0;
    uint32_t ph = 0, hphase = 0;
    bool ok = true;
    for (int phase = 1; phase <= 2 && ok; ++phase) {
      const int ub = phase == 1 ? pl.b1 : pl.b2, ue = phase == 1 ? pl.e1 : pl.e2;
      if (ub >= ue) continue;
      const int per = phase == 1 ? pl.nH : pl.tpr2;       // tiles per block
      const int runlen = phase == 1 ? pl.tpe1 : pl.nI;    // tiles per contiguous run
      int blk_end = min(ue, (ub / per + 1) * per);
      int run_left = runlen - ub % runlen;
      int gk = ub % pl.nH;                                // K group of the next tile (phase 1)
      for (int u = ub; u < ue && ok; ++it) {
        const int n = min(kTilesPerStage, min(ue - u, run_left));
        if (!warp_wait(&s.full[st], ph, abort)) { ok = false; break; }
        if (phase == 2) {
          if (!warp_wait(&s.hfull[st], (hphase >> st) & 1, abort)) { ok = false; break; }
          hphase ^= 1u << st;
        }
        if (lane == 0 && cw == 0 && it < 8) trace_clk(P, 16 + it);
        const uint8_t* sw = stage_w(st);
        const uint16_t* ss = reinterpret_cast<const uint16_t*>(stage_s(st));
        const uint8_t* sh = stage_h(st);
        // B operand and group records of tile i of the stage
        auto bsrc = [&](int i, const uint8_t*& bcol, int& cs, const uint8_t*& rec) {
          if (phase == 1) {
            int gi = gk + i;
            while (gi >= pl.nH) gi -= pl.nH;
            bcol = xq + gi * kGroup;
            cs = xcs;
            rec = xrec + gi * 4 * C::NB * 16;
          } else {
            bcol = sh + i * C::kHTile;
            cs = kHCol;
            rec = bcol + C::kCols * kHCol;
          }
        };
        // The MMAs of up to kDepth tiles are issued before the first of them is finished (four
        // with up to four tokens; fewer with more tokens, whose accumulators take more registers).
        constexpr int kDepth = C::NB == 1 ? 4 : (C::NB == 2 ? 2 : 1);
        TileAcc<C::NB> acc[kDepth];
        for (int i0 = 0; i0 < n && ok; i0 += kDepth) {
#pragma unroll
          for (int d = 0; d < kDepth; ++d)
            if (i0 + d < n) {
              const uint8_t* bcol;
              const uint8_t* rec;
              int cs;
              bsrc(i0 + d, bcol, cs, rec);
              tile_issue<C::NB>(sw + (i0 + d) * kTileBytes, ss + (i0 + d) * kRowBlock, bcol, cs, rec, r0, kh, g, c, T,
                                acc[d]);
            }
#pragma unroll
          for (int d = 0; d < kDepth; ++d) {
            const int i = i0 + d;
            if (i >= n) break;
            tile_finish<C::NB>(acc[d], seg);
            if (u + i + 1 == blk_end) {
              const int b = nblk & 1;
              if (nblk >= 2 && !warp_wait(&s.redempty[b], ((nblk >> 1) - 1) & 1, abort)) { ok = false; break; }
#pragma unroll
              for (int nb = 0; nb < C::NB; ++nb) {
                const int t = 4 * nb + c;
                if (t < T) {
                  s.red[b][kh][t][r0] = seg[nb][0];
                  s.red[b][kh][t][r0 + 8] = seg[nb][1];
                }
                seg[nb][0] = 0.f;
                seg[nb][1] = 0.f;
              }
              __syncwarp();
              if (lane == 0) tc::mbar_arrive(&s.redfull[b]);
              ++nblk;
              blk_end = min(ue, blk_end + per);
            }
          }
        }
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&s.empty[st]);
        if (lane == 0 && cw == 0 && it < 8) trace_clk(P, 24 + it);
        u += n;
        gk += n;
        while (gk >= pl.nH) gk -= pl.nH;
        run_left -= n;
        if (run_left == 0) run_left = runlen;
        if (++st == NS) { st = 0; ph ^= 1; }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue warps
    // epilogue warp ew takes the blocks written to block-sum buffer ew (every other block), so
    // the reductions of consecutive blocks run side by side: half sums -> this CTA's partial; the
    // arrival that completes a block does its reduction (h of a feature block, or an output row
    // block), tokens in chunks of C::TC.
    constexpr int TC = C::TC;
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
        float* part = (phase == 1 ? P.p1 : P.p2) + (size_t)(key + cta) * T * kRowBlock;
        for (int t = 0; t < T; ++t)
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
          float wt = 0.f;
          if (lane < T) wt = route_weight(s.rs, P, lane, s.rs.act[j]);
          uint8_t* ht = P.hbuf + ((size_t)j * nI + fb) * C::kHTile;
          const int Rg = j * 2 * nI + fb, Ru = Rg + nI;
          for (int t0 = 0; t0 < T; t0 += TC) {
            float gs[4][TC], us[4][TC];
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
              for (int i = 0; i < TC; ++i) { gs[q][i] = 0.f; us[q][i] = 0.f; }
            sum_partials2<TC, (TC == 1 ? 4 : 1)>(P.p1, Rg, pl.first1(Rg), pl.last1(Rg), gs, Ru, pl.first1(Ru),
                                                  pl.last1(Ru), us, T, t0, lane);
#pragma unroll
            for (int i = 0; i < TC; ++i) {
              const int t = t0 + i;
              if (t < T) {
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

template <int TT>
size_t smem_fixed(int H) {
  using C = Cfg<TT>;
  return sizeof(MSmem<TT>) + (size_t)C::kCols * (H + kColPad) + (size_t)(H / kGroup) * 4 * C::NB * 16 + 128;
}

template <int TT>
int stages_tt(int H) {
  const long avail = (long)kSmemLimit - (long)smem_fixed<TT>(H);
  return (int)std::min<long>(kMMaxStages, avail > 0 ? avail / Cfg<TT>::kStageBytes : 0);
}

template <int TT>
int launch_tt(const DecParams& P0, const DecMaps& M, int grid, cudaStream_t s) {
  DecParams P = P0;
  P.nstages = stages_tt<TT>(P.H);
  const size_t smem = smem_fixed<TT>(P.H) + (size_t)P.nstages * Cfg<TT>::kStageBytes;
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
