// Plain CPU oracle for the fused grouped W4A16 mixture-of-experts FFN layer.
//
// TEST INFRASTRUCTURE ONLY. This file is the slow, obviously-correct definition that the CUDA
// path is checked against. Only the tests, the smoke check and the benchmark's CPU-baseline leg
// and reference arm may load it; the product library never links, loads or calls it, and this file
// includes nothing from the product tree.
//
// Source of the method: "Every Expert Counts: ExactMoE for Memory-Efficient W4A16 Inference"
// (mlsanity.com/paper/2608.15383, Abstract). The abstract fixes: symmetric group-128 four-bit
// weight quantisation of the routed experts only, an unchanged top-k router kept in BF16,
// execution of every selected expert (none pruned or substituted) through a GPU slot cache
// and fused grouped kernels. The quantiser formula (scale = max|w|/7,
// q = clamp(round(w/scale), -8, 7), two nibbles per byte), the renormalised top-k weights and
// the tie rule are the benchmark spec's; the rest are readings listed beside each function.
//
// Precision. Integer decisions (the scale, the codes, the top-k choice) are taken in fp32 / on
// the bf16 values exactly, as the kernels take them. All other floating point is computed in
// fp64 and returned as fp32.
//
// Every function below is pinned by tests under tests/ against closed forms, brute force,
// hand-worked fixtures (tests/golden/) and library routines.

#include <cstdint>
#include <cstring>
#include <cmath>
#include <cstdlib>
#include <vector>
#include <algorithm>
#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

constexpr int kGroup = 128;          // quantisation group along K (the abstract's "group-128")
constexpr int kRowBlock = 128;       // N must be a multiple of this (the kernels' row blocks)
constexpr int kRowGroup = 8;         // rows per packed chunk
constexpr int kChunkBytes = kRowGroup * kGroup / 2;   // 512 bytes of codes per chunk

float bf16_to_f32(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

// Round-to-nearest-even conversion fp32 -> bf16 (NaN kept quiet).
uint16_t f32_to_bf16(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu) != 0) return (uint16_t)((u >> 16) | 0x40);
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7fffu + lsb;
  return (uint16_t)(u >> 16);
}

// ---- packed layout index map (layout "MW4T v2", our own design) ----
// A matrix W[N][K] (N, K multiples of 128) is cut into row groups of 8 rows (R = n/8) and K
// groups of 128 (g = k/128, the quantisation groups; G = K/128). The codes of row group R and K
// group g are one 512-byte chunk at byte (R*G + g) * 512, so the chunks of one row group over
// all of K follow each other. Inside a chunk, the 128 K values of a row are split into four
// quarters of 32; quarter kq of row r8 = n%8 is the 16-byte piece at kq*128 + r8*16. Inside the
// piece, K values 8w..8w+7 form little-endian 32-bit word w; element e of that word
// (e = 2p + h) sits in the nibble at bit 16*h + 4*p. Each nibble holds the offset-binary code
// c = q + 8, so every byte holds two codes.
size_t code_offset(int N, int K, int n, int k, int* shift) {
  (void)N;
  const int G = K / kGroup;
  const int R = n / kRowGroup, r8 = n % kRowGroup;
  const int g = k / kGroup, kk = k % kGroup;
  const int kq = kk / 32;
  const int w = (kk % 32) / 8;
  const int e = kk % 8;
  const int p = e / 2, h = e % 2;
  const int bit = 16 * h + 4 * p;
  *shift = bit % 8;
  return ((size_t)R * G + g) * kChunkBytes + (size_t)kq * 128 + (size_t)r8 * 16 + (size_t)w * 4 + bit / 8;
}

// Scales follow the same chunk order: scale(n, g) at ((R*G + g)*8 + r8).
size_t scale_index(int K, int n, int g) {
  const int G = K / kGroup;
  return ((size_t)(n / kRowGroup) * G + g) * kRowGroup + (n % kRowGroup);
}

int code_at(const uint8_t* packed, int N, int K, int n, int k) {
  int sh;
  size_t off = code_offset(N, K, n, k, &sh);
  return (packed[off] >> sh) & 0xF;
}

// Dequantised weight w_hat(n, k) = q * s, exact in fp32 and fp64.
double weight_at(const uint8_t* packed, const uint16_t* scales, int N, int K, int n, int k) {
  const int q = code_at(packed, N, K, n, k) - 8;
  const double s = (double)bf16_to_f32(scales[scale_index(K, n, k / kGroup)]);
  return (double)q * s;
}

void decode_row(const uint8_t* packed, const uint16_t* scales, int N, int K, int n, double* row) {
  for (int k = 0; k < K; ++k) row[k] = weight_at(packed, scales, N, K, n, k);
}

double silu(double z) { return z / (1.0 + std::exp(-z)); }

bool shape_ok(int N, int K) { return N > 0 && K > 0 && N % kRowBlock == 0 && K % kGroup == 0; }

}  // namespace

extern "C" {

float orc_bf16_to_f32(uint16_t b) { return bf16_to_f32(b); }
uint16_t orc_f32_to_bf16(float f) { return f32_to_bf16(f); }

size_t orc_packed_bytes(int N, int K) { return (size_t)N * K / 2; }
size_t orc_scale_count(int N, int K) { return (size_t)N * (K / kGroup); }

// Symmetric group-128 int4 quantisation (ExactMoE abstract; formula of the benchmark spec).
// For each row n and group g of 128 consecutive K elements, with w the bf16 values read
// exactly as fp32:
//   a = max |w|;  s = bf16_rne(a / 7) (fp32 IEEE division);  q = clamp(rint(w / float(s)), -8, 7)
// where rint rounds half to even and the division is fp32 IEEE. A group whose stored scale is
// zero (all-zero group, or a/7 below the bf16 range) gets q = 0.
// Outputs: q[N][K] int8 row-major, s[N][K/128] bf16 bits row-major.
int orc_quantize(const uint16_t* w, int N, int K, int8_t* q, uint16_t* s) {
  if (!w || !q || !s || !shape_ok(N, K)) return 1;
  const int G = K / kGroup;
  for (int n = 0; n < N; ++n) {
    for (int g = 0; g < G; ++g) {
      const uint16_t* wg = w + (size_t)n * K + (size_t)g * kGroup;
      float a = 0.0f;
      for (int i = 0; i < kGroup; ++i) a = std::max(a, std::fabs(bf16_to_f32(wg[i])));
      const float s32 = a / 7.0f;
      const uint16_t sb = f32_to_bf16(s32);
      const float sf = bf16_to_f32(sb);
      s[(size_t)n * G + g] = sb;
      int8_t* qg = q + (size_t)n * K + (size_t)g * kGroup;
      for (int i = 0; i < kGroup; ++i) {
        if (sf == 0.0f) { qg[i] = 0; continue; }
        const float r = std::nearbyint(bf16_to_f32(wg[i]) / sf);
        qg[i] = (int8_t)std::min(7.0f, std::max(-8.0f, r));
      }
    }
  }
  return 0;
}

// Packs q[N][K] (values -8..7) and row-major scales s[N][K/128] into the chunked layout
// described at code_offset() / scale_index().
int orc_pack(const int8_t* q, const uint16_t* s, int N, int K, uint8_t* packed, uint16_t* scales_packed) {
  if (!q || !s || !packed || !scales_packed || !shape_ok(N, K)) return 1;
  const int G = K / kGroup;
  std::memset(packed, 0, orc_packed_bytes(N, K));
  for (int n = 0; n < N; ++n)
    for (int k = 0; k < K; ++k) {
      const int qv = q[(size_t)n * K + k];
      if (qv < -8 || qv > 7) return 1;
      int sh;
      const size_t off = code_offset(N, K, n, k, &sh);
      packed[off] |= (uint8_t)((qv + 8) << sh);
    }
  for (int n = 0; n < N; ++n)
    for (int g = 0; g < G; ++g) scales_packed[scale_index(K, n, g)] = s[(size_t)n * G + g];
  return 0;
}

// Inverse of orc_pack: recovers q[N][K] and row-major scales s[N][K/128].
int orc_unpack(const uint8_t* packed, const uint16_t* scales_packed, int N, int K, int8_t* q, uint16_t* s) {
  if (!packed || !scales_packed || !q || !s || !shape_ok(N, K)) return 1;
  const int G = K / kGroup;
  for (int n = 0; n < N; ++n)
    for (int k = 0; k < K; ++k) q[(size_t)n * K + k] = (int8_t)(code_at(packed, N, K, n, k) - 8);
  for (int n = 0; n < N; ++n)
    for (int g = 0; g < G; ++g) s[(size_t)n * G + g] = scales_packed[scale_index(K, n, g)];
  return 0;
}

// Dequantises a packed matrix to fp32: out[N][K] = q * s (exact).
int orc_dequant(const uint8_t* packed, const uint16_t* scales_packed, int N, int K, float* out) {
  if (!packed || !scales_packed || !out || !shape_ok(N, K)) return 1;
  for (int n = 0; n < N; ++n)
    for (int k = 0; k < K; ++k) out[(size_t)n * K + k] = (float)weight_at(packed, scales_packed, N, K, n, k);
  return 0;
}

// Unchanged top-k routing (ExactMoE abstract: "unchanged top-k routing procedure", router in
// BF16). For each token the experts are ordered by (bf16 logit descending, expert id
// ascending) and the first k are selected; the bf16 values are compared exactly, so -0 and +0
// tie. Softmax over all E logits (fp64 here), then the k selected probabilities are
// renormalised to sum to one. idx[T][k] int32, wts[T][k] fp32.
int orc_route(const uint16_t* logits, int T, int E, int k, int32_t* idx, float* wts) {
  if (!logits || !idx || !wts || T < 0 || E <= 0 || k <= 0 || k > E) return 1;
  std::vector<float> l(E);
  std::vector<char> taken(E);
  std::vector<double> p(E);
  for (int t = 0; t < T; ++t) {
    for (int e = 0; e < E; ++e) l[e] = bf16_to_f32(logits[(size_t)t * E + e]);
    std::fill(taken.begin(), taken.end(), 0);
    for (int j = 0; j < k; ++j) {
      int best = -1;
      for (int e = 0; e < E; ++e) {
        if (taken[e]) continue;
        if (best < 0 || l[e] > l[best]) best = e;   // strict '>' keeps the lower id on ties
      }
      taken[best] = 1;
      idx[(size_t)t * k + j] = best;
    }
    double m = -INFINITY;
    for (int e = 0; e < E; ++e) m = std::max(m, (double)l[e]);
    double z = 0.0;
    for (int e = 0; e < E; ++e) { p[e] = std::exp((double)l[e] - m); z += p[e]; }
    for (int e = 0; e < E; ++e) p[e] /= z;
    double sel = 0.0;
    for (int j = 0; j < k; ++j) sel += p[idx[(size_t)t * k + j]];
    for (int j = 0; j < k; ++j) wts[(size_t)t * k + j] = (float)(p[idx[(size_t)t * k + j]] / sel);
  }
  return 0;
}

// Groups the (token, choice) pairs by expert (the "grouped" execution of the abstract).
// counts[e] = number of pairs routed to e; offsets[E+1] = exclusive prefix sum;
// perm[p] = pair id t*k + j of the p-th pair in (expert, token, choice) order;
// inv[t*k + j] = p.
int orc_permute(const int32_t* idx, int T, int k, int E, int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv) {
  if (!idx || !counts || !offsets || !perm || !inv || T < 0 || k <= 0 || E <= 0) return 1;
  for (int e = 0; e < E; ++e) counts[e] = 0;
  for (int i = 0; i < T * k; ++i) {
    if (idx[i] < 0 || idx[i] >= E) return 1;
    counts[idx[i]]++;
  }
  offsets[0] = 0;
  for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
  int pos = 0;
  for (int e = 0; e < E; ++e)
    for (int t = 0; t < T; ++t)
      for (int j = 0; j < k; ++j)
        if (idx[(size_t)t * k + j] == e) perm[pos++] = t * k + j;
  for (int p = 0; p < T * k; ++p) inv[perm[p]] = p;
  return 0;
}

// The MoE FFN layer output for the requested tokens:
//   y_e(x) = W2_e . ( silu(W_gate_e . x) * (W_up_e . x) ),   silu(z) = z / (1 + exp(-z))
//   out[t] = sum_{j < k, active(e_j)} wts[t][j] * y_{e_j}(x_t)
// with every W the dequantised weight q * s of the packed banks:
//   w13 packs [E][2I][H] (rows 0..I-1 gate, I..2I-1 up), w2 packs [E][H][I].
// x is bf16 [T][H]. tokens[n_tokens] lists the tokens to compute (NULL: all T, in order);
// out[n_tokens][H] fp32. active[E] (NULL: all experts) restricts the sum to a subset of
// experts, as one wave of a slot cache smaller than the routed set does. Arithmetic in fp64.
int orc_moe_ffn(const uint16_t* x, int T, int H, int I, int E, int k,
                const int32_t* idx, const float* wts,
                const uint8_t* w13, const uint16_t* s13,
                const uint8_t* w2, const uint16_t* s2,
                const int32_t* tokens, int n_tokens, const uint8_t* active,
                float* out, int n_threads) {
  if (!x || !idx || !wts || !w13 || !s13 || !w2 || !s2 || !out) return 1;
  if (!shape_ok(2 * I, H) || !shape_ok(H, I) || E <= 0 || k <= 0 || k > E || T < 0) return 1;
  const int nt = tokens ? n_tokens : T;
  const size_t w13_stride = orc_packed_bytes(2 * I, H), s13_stride = orc_scale_count(2 * I, H);
  const size_t w2_stride = orc_packed_bytes(H, I), s2_stride = orc_scale_count(H, I);
  const int n_pairs = nt * k;
  std::vector<double> y((size_t)n_pairs * H, 0.0);
#ifdef _OPENMP
  if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
  for (int pi = 0; pi < n_pairs; ++pi) {
    const int ti = pi / k, j = pi % k;
    const int t = tokens ? tokens[ti] : ti;
    const int e = idx[(size_t)t * k + j];
    if (e < 0 || e >= E) continue;
    if (active && !active[e]) continue;
    std::vector<double> xv(H), row(std::max(H, I)), h(I);
    for (int c = 0; c < H; ++c) xv[c] = bf16_to_f32(x[(size_t)t * H + c]);
    const uint8_t* pw13 = w13 + (size_t)e * w13_stride;
    const uint16_t* ps13 = s13 + (size_t)e * s13_stride;
    for (int i = 0; i < I; ++i) {
      decode_row(pw13, ps13, 2 * I, H, i, row.data());
      double g = 0.0;
      for (int c = 0; c < H; ++c) g += row[c] * xv[c];
      decode_row(pw13, ps13, 2 * I, H, I + i, row.data());
      double u = 0.0;
      for (int c = 0; c < H; ++c) u += row[c] * xv[c];
      h[i] = silu(g) * u;
    }
    const uint8_t* pw2 = w2 + (size_t)e * w2_stride;
    const uint16_t* ps2 = s2 + (size_t)e * s2_stride;
    double* yp = y.data() + (size_t)pi * H;
    for (int n = 0; n < H; ++n) {
      decode_row(pw2, ps2, H, I, n, row.data());
      double acc = 0.0;
      for (int i = 0; i < I; ++i) acc += row[i] * h[i];
      yp[n] = acc;
    }
  }
  for (int ti = 0; ti < nt; ++ti) {
    const int t = tokens ? tokens[ti] : ti;
    for (int n = 0; n < H; ++n) {
      double acc = 0.0;
      for (int j = 0; j < k; ++j) acc += (double)wts[(size_t)t * k + j] * y[((size_t)ti * k + j) * H + n];
      out[(size_t)ti * H + n] = (float)acc;
    }
  }
  return 0;
}

// The same MoE FFN layer on UNQUANTISED bf16 expert weights (the BF16 configuration the ExactMoE
// abstract compares its W4A16 decode against): w13 [E][2I][H] (rows 0..I-1 gate, I..2I-1 up) and
// w2 [E][H][I], row-major bf16, read exactly as fp32; everything else as orc_moe_ffn (fp64).
int orc_moe_ffn_bf16(const uint16_t* x, int T, int H, int I, int E, int k,
                     const int32_t* idx, const float* wts,
                     const uint16_t* w13, const uint16_t* w2,
                     const int32_t* tokens, int n_tokens, const uint8_t* active,
                     float* out, int n_threads) {
  if (!x || !idx || !wts || !w13 || !w2 || !out) return 1;
  if (H <= 0 || I <= 0 || E <= 0 || k <= 0 || k > E || T < 0) return 1;
  const int nt = tokens ? n_tokens : T;
  const size_t w13_stride = (size_t)2 * I * H, w2_stride = (size_t)H * I;
  const int n_pairs = nt * k;
  std::vector<double> y((size_t)n_pairs * H, 0.0);
#ifdef _OPENMP
  if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
  for (int pi = 0; pi < n_pairs; ++pi) {
    const int ti = pi / k, j = pi % k;
    const int t = tokens ? tokens[ti] : ti;
    const int e = idx[(size_t)t * k + j];
    if (e < 0 || e >= E) continue;
    if (active && !active[e]) continue;
    std::vector<double> xv(H), h(I);
    for (int c = 0; c < H; ++c) xv[c] = bf16_to_f32(x[(size_t)t * H + c]);
    const uint16_t* pw13 = w13 + (size_t)e * w13_stride;
    for (int i = 0; i < I; ++i) {
      double g = 0.0, u = 0.0;
      for (int c = 0; c < H; ++c) g += (double)bf16_to_f32(pw13[(size_t)i * H + c]) * xv[c];
      for (int c = 0; c < H; ++c) u += (double)bf16_to_f32(pw13[(size_t)(I + i) * H + c]) * xv[c];
      h[i] = silu(g) * u;
    }
    const uint16_t* pw2 = w2 + (size_t)e * w2_stride;
    double* yp = y.data() + (size_t)pi * H;
    for (int n = 0; n < H; ++n) {
      double acc = 0.0;
      for (int i = 0; i < I; ++i) acc += (double)bf16_to_f32(pw2[(size_t)n * I + i]) * h[i];
      yp[n] = acc;
    }
  }
  for (int ti = 0; ti < nt; ++ti) {
    const int t = tokens ? tokens[ti] : ti;
    for (int n = 0; n < H; ++n) {
      double acc = 0.0;
      for (int j = 0; j < k; ++j) acc += (double)wts[(size_t)t * k + j] * y[((size_t)ti * k + j) * H + n];
      out[(size_t)ti * H + n] = (float)acc;
    }
  }
  return 0;
}

// One wave of the GPU slot cache (the abstract's "configurable GPU-resident slot cache"; the
// pages give no policy, so this is the plainest reading: least-recently-used replacement).
// State: slot_expert[S] (-1 = free), last_used[S], *clock. needed[E] (0/1) marks the experts
// that still have to run this step; on return the experts of this wave are cleared from it.
// cap (1..S) bounds the experts of one wave; protect[S] (may be null) marks slots that must not
// be overwritten in this wave (a wave still reading them).
//   - hits = needed experts already resident, misses = the others, both in ascending id;
//   - the wave is the first min(cap, |hits|) hits plus the first cap - (hits taken) misses;
//   - each miss of the wave, in ascending id, takes the lowest free slot, else evicts the
//     slot with the smallest last_used (ties: lowest slot) that is not protected and whose
//     expert is not needed (neither in this wave nor waiting for a later one);
//   - every slot of the wave gets last_used = *clock, then *clock += 1.
// With cap = S and no protected slot every hit is in the wave and this is plain LRU.
// Outputs: wave_table[E] = slot of each expert in the wave, -1 for all others;
// loads_expert/loads_slot[*n_loads] = the misses in load order.
int orc_slot_wave_capped(int E, int S, int cap, const uint8_t* protect, int32_t* slot_expert, int64_t* last_used,
                         int64_t* clock, uint8_t* needed, int32_t* wave_table, int32_t* loads_expert,
                         int32_t* loads_slot, int* n_loads) {
  if (E <= 0 || S <= 0 || cap < 1 || cap > S || !slot_expert || !last_used || !clock || !needed || !wave_table ||
      !loads_expert || !loads_slot || !n_loads)
    return 1;
  std::vector<int> slot_of(E, -1);
  for (int s = 0; s < S; ++s)
    if (slot_expert[s] >= 0 && slot_expert[s] < E) slot_of[slot_expert[s]] = s;
  std::vector<int> hits, misses;
  for (int e = 0; e < E; ++e) {
    if (!needed[e]) continue;
    if (slot_of[e] >= 0) hits.push_back(e); else misses.push_back(e);
  }
  std::vector<char> in_wave(E, 0);
  const int n_hit = std::min(cap, (int)hits.size());
  for (int i = 0; i < n_hit; ++i) in_wave[hits[i]] = 1;
  const int n_new = std::min(cap - n_hit, (int)misses.size());
  for (int i = 0; i < n_new; ++i) in_wave[misses[i]] = 1;
  *n_loads = 0;
  for (int i = 0; i < n_new; ++i) {
    const int e = misses[i];
    int pick = -1;
    for (int s = 0; s < S; ++s)
      if (slot_expert[s] < 0) { pick = s; break; }
    if (pick < 0) {
      for (int s = 0; s < S; ++s) {
        const int old = slot_expert[s];
        if (old >= 0 && (in_wave[old] || needed[old])) continue;
        if (protect && protect[s]) continue;
        if (pick < 0 || last_used[s] < last_used[pick]) pick = s;
      }
    }
    if (pick < 0) return 2;
    if (slot_expert[pick] >= 0) slot_of[slot_expert[pick]] = -1;
    slot_expert[pick] = e;
    slot_of[e] = pick;
    loads_expert[*n_loads] = e;
    loads_slot[*n_loads] = pick;
    (*n_loads)++;
  }
  for (int e = 0; e < E; ++e) {
    wave_table[e] = in_wave[e] ? slot_of[e] : -1;
    if (in_wave[e]) {
      last_used[slot_of[e]] = *clock;
      needed[e] = 0;
    }
  }
  *clock += 1;
  return 0;
}

int orc_slot_wave(int E, int S, int32_t* slot_expert, int64_t* last_used, int64_t* clock, uint8_t* needed,
                  int32_t* wave_table, int32_t* loads_expert, int32_t* loads_slot, int* n_loads) {
  return orc_slot_wave_capped(E, S, S, nullptr, slot_expert, last_used, clock, needed, wave_table, loads_expert,
                              loads_slot, n_loads);
}

}  // extern "C"
