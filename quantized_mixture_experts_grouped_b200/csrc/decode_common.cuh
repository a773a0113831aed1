// Pieces of the fused decode kernels: in-kernel routing and the compact token lists, the
// byte-balanced split of the selected experts' packed tiles over the CTAs (batched kernel), the
// scratch and counter layout, and the deterministic cross-CTA reductions ("Every Expert Counts: ExactMoE for
// Memory-Efficient W4A16 Inference", Abstract: every selected expert runs through fused grouped
// MoE kernels; the router's top-k is unchanged).
//
// Work split. Phase 1 (gate/up) walks the selected experts' W13 tiles expert by expert in stored
// order; phase 2 (down) walks W2 tiles ordered (output row block, expert, K group). Each phase's
// tiles are divided into equal contiguous ranges, one per CTA, so that a CTA moves its weights
// in a few long bulk copies. A CTA writes one fp32 partial per 128-row block it touches; the
// CTA that completes the last partial of a block (counted with an atomic) sums the partials in
// CTA order, so results do not depend on timing.
#pragma once

#include <algorithm>
#include <cuda.h>

#include "common.cuh"
#include "tc.cuh"

namespace moe {
namespace dec {

constexpr int kMaxTk = 256;
constexpr int kMaxT = 16;
constexpr int kTilesPerStage = 4;          // one bulk copy moves up to 4 packed tiles (32 KB)
constexpr int kMaxGrid = 160;
constexpr int kStageW = kTilesPerStage * kTileBytes;
constexpr int kStageS = kTilesPerStage * kRowBlock * 2;
constexpr int kSmemLimit = 227 * 1024;
constexpr unsigned kFull = 0xffffffffu;

// status "where" codes of the decode kernels
enum { kSiteStage = 2, kSiteABuf = 3, kSiteH = 4, kSiteAcc = 5, kSiteHDone = 6, kSiteDrain = 7, kSiteOver = 8 };

struct DecParams {
  const uint16_t* x; const uint16_t* logits; const int32_t* idx_in; const float* wts_in;
  int T, H, I, E, k;
  const uint8_t* w13; const uint16_t* s13; const uint8_t* w2; const uint16_t* s2;
  const int32_t* slot;
  int32_t* idx_out; float* wts_out;
  uint16_t* out; float* acc; int accumulate;
  int* ctl;
  int* hcnt;                    // [selected expert][I/128] phase-1 arrivals per feature block
  int* fcnt;                    // [H/128] phase-2 arrivals per output row block
  int* hdone;                   // [0] feature blocks finished, [1] CTAs finished, [2..3] as u64:
                                // running count of CTAs past phase 1 (single-token kernel)
  float* p1;                    // phase-1 partials: [row block + CTA][T][128]
  float* p2;                    // phase-2 partials: [output block + CTA][T][128]
  uint8_t* hbuf;                // h operand tiles (layout depends on the kernel)
  int nstages;
  uint32_t mul16;               // 65536, passed at run time so that x * mul16 stays an IMAD
  unsigned long long* trace;    // optional per-CTA diagnostics (64 x u64 per CTA), null normally
  long long wait_cycles;        // single-token kernel: limit of its bounded waits (0 = default)
  int extra_arrivals;           // single-token kernel: arrivals expected beyond the grid (test hook)
};

// Tensor maps of the two packed banks, one 128 x 128 tile per box (make_chunk_code_map).
struct alignas(64) DecMaps {
  CUtensorMap c13, s13, c2, s2;
};

// trace slots per CTA: 0 start, 1 plan done, 3 weights all issued, 4 all h ready, 5 compute
// done, 6 end (%globaltimer); 7 SM clock after the plan; 8..11 values; 12.. SM clock stamps
__device__ __forceinline__ void trace_at(const DecParams& P, int slot) {
  if (P.trace) P.trace[blockIdx.x * 64 + slot] = tc::globaltimer();
}
__device__ __forceinline__ void trace_val(const DecParams& P, int slot, long long v) {
  if (P.trace) P.trace[blockIdx.x * 64 + slot] = (unsigned long long)v;
}
__device__ __forceinline__ void trace_clk(const DecParams& P, int slot) {
  if (P.trace) P.trace[blockIdx.x * 64 + slot] = (unsigned long long)clock64();
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
  const bool ok = tc::mbar_wait(bar, parity, abort);
  return __all_sync(kFull, ok);
}

__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

__device__ __forceinline__ void ffma2(float& dx, float& dy, float ax, float ay, float bx, float by) {
  unsigned long long d, a, b, c;
  asm("mov.b64 %0, {%1, %2};" : "=l"(a) : "f"(ax), "f"(ay));
  asm("mov.b64 %0, {%1, %2};" : "=l"(b) : "f"(bx), "f"(by));
  asm("mov.b64 %0, {%1, %2};" : "=l"(c) : "f"(dx), "f"(dy));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(dx), "=f"(dy) : "l"(d));
}

// Routing state kept in shared memory by both kernels.
struct RouteSmem {
  int idx[kMaxTk];
  float wts[kMaxTk];
  uint32_t present[kMaxExperts / 32];
  uint32_t tokbits[kMaxT][kMaxExperts / 32];
  int act[kMaxExperts];
  int sl[kMaxExperts];      // slot of act[j]
  uint8_t ntok[kMaxExperts];            // tokens routed to act[j]
  uint8_t tok[kMaxExperts][kMaxT];      // ... in ascending order (the expert's compact token list)
  int nact;
  int over;
};

__device__ __forceinline__ uint32_t route_key(uint32_t bits, int e) {
  bits &= 0xffffu;
  if (bits == 0x8000u) bits = 0;
  const uint32_t ord = (bits & 0x8000u) ? (~bits & 0xffffu) : (bits | 0x8000u);
  return (ord << 16) | (0xffffu - (uint32_t)e);
}

// Routes token t with one warp (same selection rule as the stand-alone router: bf16 logit
// descending, expert id ascending). Lane l holds the keys of experts l, l+32, ...; each of the
// k rounds takes the warp maximum of the keys (unique: the id is in them) and retires it. The
// chosen logits are decoded back from the winning keys; the renormalised weight of choice j is
// exp(l_j - l_max) / sum over the k chosen (= the full softmax renormalised over the chosen),
// with the exponentials taken after the selection, one per lane.
template <int kPer>
__device__ inline void route_token_n(RouteSmem& rs, const DecParams& P, int t, int lane) {
  const int E = P.E, k = P.k;
  const uint16_t* lt = P.logits + (size_t)t * E;
  uint32_t key[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int e = lane + 32 * i;
    key[i] = (e < E) ? route_key(lt[e], e) : 0u;
  }
  uint32_t mine[8];    // lane (j % 32) keeps the winning key of choice j in mine[j / 32]
#pragma unroll
  for (int i = 0; i < 8; ++i) mine[i] = 0;
  uint32_t first = 0;
  for (int j = 0; j < k; ++j) {
    uint32_t best = key[0];
#pragma unroll
    for (int i = 1; i < kPer; ++i) best = max(best, key[i]);
    const uint32_t win = __reduce_max_sync(kFull, best);
#pragma unroll
    for (int i = 0; i < kPer; ++i)
      if (key[i] == win) key[i] = 0;
    if (j == 0) first = win;
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if ((j & 31) == lane && (j >> 5) == i) mine[i] = win;
  }
  auto logit_of = [](uint32_t w) {
    const uint32_t ord = w >> 16;
    return bf16_bits_to_float((ord & 0x8000u) ? (ord & 0x7fffu) : (~ord & 0xffffu));
  };
  const float mx = logit_of(first);
  float el[8], sum = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {   // rounds past k are skipped (a uniform branch)
    el[i] = 0.f;
    if (32 * i >= k) continue;
    const int j = 32 * i + lane;
    if (j < k) {
      el[i] = expf(logit_of(mine[i]) - mx);
      rs.idx[t * k + j] = 0xffff - (int)(mine[i] & 0xffffu);
    }
    sum += el[i];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(kFull, sum, o);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    if (32 * i >= k) continue;
    const int j = 32 * i + lane;
    if (j < k) rs.wts[t * k + j] = el[i] / sum;
  }
}

__device__ inline void route_token(RouteSmem& rs, const DecParams& P, int t, int lane) {
  if (P.E <= 64) route_token_n<2>(rs, P, t, lane);
  else if (P.E <= 128) route_token_n<4>(rs, P, t, lane);
  else route_token_n<8>(rs, P, t, lane);
}

// Clears the routing state (before the dependency wait; no global reads).
__device__ inline void route_clear(RouteSmem& rs, int tid, int nthreads) {
  for (int i = tid; i < kMaxExperts / 32; i += nthreads) rs.present[i] = 0;
  for (int i = tid; i < kMaxT * kMaxExperts / 32; i += nthreads) (&rs.tokbits[0][0])[i] = 0;
  if (tid == 0) rs.over = 0;
}

// Routing (or the given routing) into shared memory. Call with every thread of the CTA,
// followed by __syncthreads() and route_finish().
__device__ inline void route_begin(RouteSmem& rs, const DecParams& P, int tid, int nthreads) {
  const int warp = tid >> 5, lane = tid & 31;
  if (P.logits) {
    for (int t = warp; t < P.T; t += nthreads / 32) route_token(rs, P, t, lane);
  } else {
    for (int p = tid; p < P.T * P.k; p += nthreads) {
      rs.idx[p] = P.idx_in[p];
      rs.wts[p] = P.wts_in[p];
    }
  }
}

// Presence bitmap, duplicate check, selected experts in ascending id. Contains two CTA barriers.
__device__ inline void route_finish(RouteSmem& rs, const DecParams& P, int tid, int nthreads) {
  const int Tk = P.T * P.k, E = P.E;
  for (int p = tid; p < Tk; p += nthreads) {
    const int e = rs.idx[p], t = p / P.k;
    if ((unsigned)e >= (unsigned)E || slot_of(P.slot, e) < 0) continue;   // not resident: skipped
    atomicOr(&rs.present[e >> 5], 1u << (e & 31));
    const uint32_t old = atomicOr(&rs.tokbits[t][e >> 5], 1u << (e & 31));
    if ((old >> (e & 31)) & 1u) rs.over = 1;     // a token routed twice to one expert
  }
  if (P.logits && P.idx_out && blockIdx.x == 0)
    for (int p = tid; p < Tk; p += nthreads) {
      P.idx_out[p] = rs.idx[p];
      P.wts_out[p] = rs.wts[p];
    }
  __syncthreads();
  if (tid < E) {   // rank = set bits below in the presence bitmap
    const int w = tid >> 5;
    if ((rs.present[w] >> (tid & 31)) & 1u) {
      int a = __popc(rs.present[w] & ((1u << (tid & 31)) - 1u));
      for (int i = 0; i < w; ++i) a += __popc(rs.present[i]);
      rs.act[a] = tid;
      rs.sl[a] = slot_of(P.slot, tid);
      int n = 0;
      for (int t = 0; t < P.T; ++t)
        if ((rs.tokbits[t][w] >> (tid & 31)) & 1u) rs.tok[a][n++] = (uint8_t)t;
      rs.ntok[a] = (uint8_t)n;
    }
  }
  if (tid == 0) {
    int n = 0;
    for (int i = 0; i < (E + 31) / 32; ++i) n += __popc(rs.present[i]);
    rs.nact = rs.over ? 0 : n;
    if (rs.over) report_status(P.ctl, MOE_ERR_ARG, kSiteOver);
  }
  __syncthreads();
}

// Router weight of selected expert e for token t (0 if the token does not route to it).
__device__ __forceinline__ float route_weight(const RouteSmem& rs, const DecParams& P, int t, int e) {
  float w = 0.f;
  for (int q = 0; q < P.k; ++q)
    if (rs.idx[t * P.k + q] == e) w = rs.wts[t * P.k + q];
  return w;
}

// The static split of the selected experts' tiles over the CTAs, identical in every CTA. Phase
// p uses the first Gp = min(grid, tiles) CTAs, so every one of them has a non-empty range.
struct Plan {
  int m, nI, nH;
  int tpe1;             // W13 tiles per expert (2I/128 row blocks x H/128 K groups)
  int tpr2;             // W2 tiles per output row block (m experts x I/128 K groups)
  int n1, n2;           // tiles of each phase
  int G1, G2;
  int b1, e1, b2, e2;   // this CTA's tile ranges
  // 32-bit arithmetic: the host only launches when tiles x grid < 2^32 (split_fits)
  __device__ static int start(int c, int n, int G) { return G ? (int)(((uint32_t)c * (uint32_t)n) / (uint32_t)G) : 0; }
  __device__ static int owner(int u, int n, int G) {
    return (int)(((uint32_t)(u + 1) * (uint32_t)G - 1u) / (uint32_t)n);
  }
  __device__ void init(int m_, int H, int I, int G, int c) {
    m = m_; nI = I / kRowBlock; nH = H / kGroup;
    tpe1 = 2 * nI * nH;
    tpr2 = m * nI;
    n1 = m * tpe1;
    n2 = nH * tpr2;
    G1 = min(G, n1);
    G2 = min(G, n2);
    b1 = c < G1 ? start(c, n1, G1) : 0; e1 = c < G1 ? start(c + 1, n1, G1) : 0;
    b2 = c < G2 ? start(c, n2, G2) : 0; e2 = c < G2 ? start(c + 1, n2, G2) : 0;
  }
  // tiles of the stage that starts at tile u (a run stays inside one contiguous stored block)
  __device__ int run1(int u) const { return min(kTilesPerStage, min(e1 - u, tpe1 - u % tpe1)); }
  __device__ int run2(int u) const { return min(kTilesPerStage, min(e2 - u, nI - u % nI)); }
  // CTAs holding a part of phase-1 row block R (tiles R*nH ..) / phase-2 output block ob
  __device__ int first1(int R) const { return owner(R * nH, n1, G1); }
  __device__ int last1(int R) const { return owner((R + 1) * nH - 1, n1, G1); }
  __device__ int first2(int ob) const { return owner(ob * tpr2, n2, G2); }
  __device__ int last2(int ob) const { return owner((ob + 1) * tpr2 - 1, n2, G2); }
  // global memory of the stage starting at tile u of a phase: expert slot index j, tile index
  __device__ void locate(int phase, int u, int& j, int& lt) const {
    if (phase == 1) {
      j = u / tpe1; lt = u % tpe1;
    } else {
      const int ob = u / tpr2, rem = u % tpr2;
      j = rem / nI; lt = ob * nI + rem % nI;
    }
  }
};

// Arrival of one CTA's partial of block `key` (phase 1: W13 row block, phase 2: output block).
// Returns true for the arrival that completes the block (its counter is reset for the next
// launch). Called by one thread after the partial's stores were fenced.
__device__ inline bool block_arrive(const Plan& pl, const DecParams& P, int phase, int key) {
  int* cnt;
  int target;
  if (phase == 1) {
    const int nI = pl.nI, j = key / (2 * nI), fb = (key % (2 * nI)) % nI;
    const int Rg = j * 2 * nI + fb, Ru = Rg + nI;
    cnt = P.hcnt + j * nI + fb;
    target = (pl.last1(Rg) - pl.first1(Rg) + 1) + (pl.last1(Ru) - pl.first1(Ru) + 1);
  } else {
    cnt = P.fcnt + key;
    target = pl.last2(key) - pl.first2(key) + 1;
  }
  int old;   // acquire-release: publishes this CTA's partial, and makes the others' visible
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], 1;" : "=r"(old) : "l"(cnt) : "memory");
  if (old != target - 1) return false;
  *cnt = 0;
  __threadfence();
  return true;
}

// Gate and up sums of feature r of feature block fb of selected expert j (phase-1 partials in
// CTA order), for tokens t < T, into g[] and u[].
template <int TN>
__device__ __forceinline__ void gate_up_sums(const Plan& pl, const DecParams& P, int j, int fb, int r,
                                             float (&g)[TN], float (&u)[TN]) {
  const int nI = pl.nI, Rg = j * 2 * nI + fb, Ru = Rg + nI, T = P.T;
#pragma unroll
  for (int t = 0; t < TN; ++t) { g[t] = 0.f; u[t] = 0.f; }
  for (int c = pl.first1(Rg); c <= pl.last1(Rg); ++c) {
    const float* pp = P.p1 + (size_t)(Rg + c) * T * kRowBlock + r;
#pragma unroll
    for (int t = 0; t < TN; ++t)
      if (t < T) g[t] += __ldcg(pp + t * kRowBlock);
  }
  for (int c = pl.first1(Ru); c <= pl.last1(Ru); ++c) {
    const float* pp = P.p1 + (size_t)(Ru + c) * T * kRowBlock + r;
#pragma unroll
    for (int t = 0; t < TN; ++t)
      if (t < T) u[t] += __ldcg(pp + t * kRowBlock);
  }
}

__device__ __forceinline__ float swiglu(float g, float u) { return g / (1.f + expf(-g)) * u; }

// Output element (t, n) from its fp32 sum y: added to the fp32 accumulator (wave accumulation)
// and either stored back there (no output given) or rounded to the bf16 output.
__device__ __forceinline__ void store_output(const DecParams& P, int t, int n, float y) {
  const size_t o = (size_t)t * P.H + n;
  const float accv = (P.accumulate ? __ldcg(P.acc + o) : 0.f) + y;
  if (P.out) {
    P.out[o] = __bfloat16_as_ushort(__float2bfloat16_rn(accv));
    if (P.accumulate) P.acc[o] = 0.f;
  } else {
    P.acc[o] = accv;
  }
}

// Output row block `ob` (row r of it): the phase-2 partials summed in CTA order, then the
// combine with the fp32 accumulator (wave accumulation) and the bf16 output.
template <int TN>
__device__ __forceinline__ void output_block(const Plan& pl, const DecParams& P, int ob, int r) {
  const int T = P.T;
  float y[TN];
#pragma unroll
  for (int t = 0; t < TN; ++t) y[t] = 0.f;
  for (int c = pl.first2(ob); c <= pl.last2(ob); ++c) {
    const float* pp = P.p2 + (size_t)(ob + c) * T * kRowBlock + r;
#pragma unroll
    for (int t = 0; t < TN; ++t)
      if (t < T) y[t] += __ldcg(pp + t * kRowBlock);
  }
#pragma unroll
  for (int t = 0; t < TN; ++t)
    if (t < T) store_output(P, t, ob * kRowBlock + r, y[t]);
}

// End of a decode launch, every thread: outputs when no expert was selected, then the last CTA
// to leave resets the counters that every CTA reads.
__device__ inline void finish_launch(const Plan& pl, const DecParams& P, volatile int* abort, int tid,
                                     int nthreads) {
  if (pl.n2 == 0 && !*abort) {
    const int total = P.T * P.H;
    for (int o = blockIdx.x * nthreads + tid; o < total; o += gridDim.x * nthreads) {
      const float accv = P.accumulate ? __ldcg(P.acc + o) : 0.f;
      if (P.out) {
        P.out[o] = __bfloat16_as_ushort(__float2bfloat16_rn(accv));
        if (P.accumulate) P.acc[o] = 0.f;
      } else {
        P.acc[o] = accv;
      }
    }
  }
  if (tid == 0) {
    __threadfence();
    if (atomicAdd(P.hdone + 1, 1) == (int)gridDim.x - 1) {
      P.hdone[0] = 0;
      P.hdone[1] = 0;
      __threadfence();
    }
    trace_at(P, 6);
  }
}

// ---- warp-level int8 MMA pieces (decode kernels on the mma.sync path)
// D (16 x 8, s32) += A (16 x 32, u8) * B (32 x 8, s8).
__device__ __forceinline__ void imma(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                     uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Byte position of element e (0..7) of a word in the permuted order (0, 4, 1, 5, 2, 6, 3, 7).
__device__ __forceinline__ int perm_pos(int e) { return ((e & 3) << 1) | (e >> 2); }

// Encodes one 128-element group of one token as two B-operand columns. Lane l holds elements
// q * 32 + l (q = 0..3) in v[q]. hi / lo: the columns (bytes), starting at the group's first
// word; rec: the group's record {8 * sum(v) over elements 0..63, a, 8 * sum(v) over 64..127, a}.
// Called by a whole warp; generic pointers (shared or global memory).
__device__ __forceinline__ void encode_group(const float (&v)[4], uint8_t* hi, uint8_t* lo, int4* rec, int lane) {
  float mx = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, o));
  const float inv = mx > 0.f ? 32639.f / mx : 0.f;
  int sum0 = 0, sum1 = 0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int iv = max(-32639, min(32639, __float2int_rn(v[q] * inv)));
    const int h8 = (iv + 128) >> 8, l8 = iv - 256 * h8;
    const int k = q * 32 + lane, at = (k >> 3) * 8 + perm_pos(k & 7);
    hi[at] = (uint8_t)h8;
    lo[at] = (uint8_t)l8;
    if (q < 2) sum0 += iv; else sum1 += iv;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    sum0 += __shfl_xor_sync(kFull, sum0, o);
    sum1 += __shfl_xor_sync(kFull, sum1, o);
  }
  if (lane == 0) {
    const int a = __float_as_int(mx * (1.f / 32639.f));
    *rec = make_int4(8 * sum0, a, 8 * sum1, a);
  }
}

// The same encoding with lane l holding elements 4 l .. 4 l + 3 of the group in v[0..3] (one
// 8-byte load per lane); the columns and the record are identical to encode_group's.
__device__ __forceinline__ void encode_group_c(const float (&v)[4], uint8_t* hi, uint8_t* lo, int4* rec, int lane) {
  float mx = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, o));
  const float inv = mx > 0.f ? 32639.f / mx : 0.f;
  int sum = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int iv = max(-32639, min(32639, __float2int_rn(v[i] * inv)));
    const int h8 = (iv + 128) >> 8, l8 = iv - 256 * h8;
    const int at = (lane >> 1) * 8 + 2 * i + (lane & 1);   // element 4 lane + i, permuted in its 8-group
    hi[at] = (uint8_t)h8;
    lo[at] = (uint8_t)l8;
    sum += iv;
  }
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) sum += __shfl_xor_sync(kFull, sum, o);   // lanes 0..15 / 16..31
  const int sum1 = __shfl_sync(kFull, sum, 16);
  if (lane == 0) {
    const int a = __float_as_int(mx * (1.f / 32639.f));
    *rec = make_int4(8 * sum, a, 8 * sum1, a);
  }
}

// ---- host side
// Counters (zero between launches), in their own workspace region whose offset does not depend
// on T: hcnt [E][I/128], fcnt [H/128], hdone [4] (m <= E selected experts at any batch size).
struct DecCounters { size_t hcnt, fcnt, hdone, total; };
inline DecCounters dec_counters(int H, int I, int E) {
  DecCounters C{};
  const size_t nI = I / kRowBlock, nH = H / kRowBlock;
  size_t off = 0;
  auto take = [&](size_t bytes) { const size_t at = off; off = align_up(off + bytes, 256); return at; };
  C.hcnt = take(sizeof(int) * (size_t)E * nI);
  C.fcnt = take(sizeof(int) * nH);
  C.hdone = take(sizeof(int) * 4);
  C.total = off;
  return C;
}

// Partials and operands (no initial value needed).
struct DecScratch { size_t p1, p2, hbuf, total; };
// hbuf_per_tile: bytes of h operand per (selected expert, K group of I)
inline DecScratch dec_scratch(int T, int H, int I, int E, int k, size_t hbuf_per_tile) {
  DecScratch D{};
  const size_t m = (size_t)std::min(E, T * k), nI = I / kRowBlock, nH = H / kRowBlock;
  size_t off = 0;
  auto take = [&](size_t bytes) { const size_t at = off; off = align_up(off + bytes, 256); return at; };
  D.p1 = take(sizeof(float) * (m * 2 * nI + kMaxGrid) * T * kRowBlock);
  D.p2 = take(sizeof(float) * (nH + kMaxGrid) * T * kRowBlock);
  D.hbuf = take(m * nI * hbuf_per_tile);
  D.total = off;
  return D;
}

// The split's 32-bit arithmetic needs (tiles of a phase) x grid < 2^32.
inline bool split_fits(int T, int H, int I, int E, int k, int grid) {
  const unsigned long long m = (unsigned long long)std::min(E, T * k);
  const unsigned long long n1 = m * 2 * (I / kRowBlock) * (H / kGroup);
  return (n1 + 1) * (unsigned long long)grid < (1ull << 32);
}

int num_sms();
extern unsigned long long* g_trace;

// Single-token decode kernel (defined in ffn_decode_rows.cu)
bool rows_supported(int T, int H, int I, int E, int k);
size_t rows_hbuf_per_tile();
int launch_decode_rows(const DecParams& P, int grid, cudaStream_t s);

// Warp-MMA decode kernel for T <= kMmaMaxT (defined in ffn_decode_mma.cu)
constexpr int kMmaMaxT = 16;
size_t mma_hbuf_per_tile(int T);
int mma_stages(int T, int H);
int launch_decode_mma(const DecParams& P, int grid, cudaStream_t s);

}  // namespace dec
}  // namespace moe
