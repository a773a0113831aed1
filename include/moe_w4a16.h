/* moe_w4a16.h — C ABI of the fused grouped W4A16 mixture-of-experts FFN layer (sm_100a).
 *
 * The operation is the MoE layer of "Every Expert Counts: ExactMoE for Memory-Efficient W4A16
 * Inference" (mlsanity.com/paper/2608.15383, Abstract): routed experts hold symmetric
 * group-128 four-bit weights; the router stays BF16 and its top-k choice is left unchanged;
 * every selected expert runs, none is pruned or substituted, none runs on the CPU; experts
 * are executed through a GPU-resident slot cache and fused grouped kernels.
 *
 * Conventions for every call below:
 *  - Shapes: T tokens, H hidden, I intermediate (one expert is a SwiGLU MLP), E experts,
 *    k experts per token. H and I are multiples of 128; 1 <= k <= E <= 256.
 *  - Matrices are "row = output feature, K = input feature" (x W^T convention). The gate/up
 *    matrix of an expert is W13 = [W_gate; W_up] with 2I rows and H columns; the down matrix
 *    W2 has H rows and I columns.
 *  - bf16 values are passed as their 16-bit patterns (uint16_t).
 *  - Pointers are device pointers owned by the caller unless a comment says "host". No call
 *    allocates device memory; scratch lives in a caller-owned workspace.
 *  - Calls are asynchronous on the given stream (a cudaStream_t; NULL = legacy default
 *    stream) and return a status: MOE_OK, or an error whose text moe_last_error_string()
 *    gives. Argument errors are reported before anything is launched.
 *  - Packed weight layout "MW4T v2" (this library's own design; the abstract stores experts
 *    in a kernel-native form without giving its bytes): a matrix W[N][K] is cut into chunks of
 *    8 rows x 128 K (one quantisation group of each of the 8 rows), 512 bytes each; the chunk
 *    of row group R = n/8 and K group g is at byte (R*K/128 + g)*512, so the chunks of one row
 *    group follow each other over all of K. Inside a chunk, quarter kq (32 K values) of row
 *    r8 = n%8 is a 16-byte piece at kq*128 + r8*16; K values 8w..8w+7 of the piece form
 *    little-endian 32-bit word w, element 2p+h sitting in the nibble at bit 16h+4p. A nibble
 *    holds the offset-binary code q+8, two codes per byte. Scales are bf16, one per (row,
 *    group of 128 K), in the same chunk order: scale(n, g) at ((n/8)*(K/128) + g)*8 + n%8.
 */
#ifndef MOE_W4A16_H
#define MOE_W4A16_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* moe_stream_t; /* same handle type as cudaStream_t */
typedef struct CUevent_st* moe_event_t;   /* same handle type as cudaEvent_t  */

enum {
  MOE_OK = 0,
  MOE_ERR_ARG = 1,      /* null pointer, negative size, k > E, workspace too small ...      */
  MOE_ERR_SHAPE = 2,    /* H or I not a multiple of 128, E > 256, unsupported size          */
  MOE_ERR_CUDA = 3,     /* a CUDA runtime call failed (text in moe_last_error_string)       */
  MOE_ERR_TIMEOUT = 4   /* a kernel's bounded wait gave up (see moe_workspace_status)       */
};

/* FFN execution paths (the `flags` argument of moe_w4a16_ffn / moe_w4a16_layer). */
enum {
  MOE_PATH_AUTO = 0,       /* fused decode kernel for small batches, grouped GEMM otherwise   */
  MOE_PATH_SIMPLE = 1,     /* CUDA-core grouped kernels (reference path, any size)            */
  MOE_PATH_DECODE = 2,     /* one fused launch (T <= 16): routing, both projections on the
                              int8 warp-MMA path, in-kernel combine                          */
  MOE_PATH_GROUPED = 3,    /* permute + tcgen05 grouped GEMMs (gate/up, down) + combine       */
  MOE_PATH_SEQUENTIAL = 4, /* one expert at a time through the same kernels (ablation)        */
  MOE_PATH_MASK = 0xff,
  MOE_FLAG_ACCUMULATE = 0x100 /* add this call's contribution into the workspace fp32
                                 accumulator instead of starting from zero (slot-cache waves) */
};

/* Version of this ABI and of the packed layout ("MW4T v2" -> 2). */
int moe_abi_version(void);
int moe_packed_layout_version(void);

/* Text of the last error reported by any call on this thread. Never NULL. */
const char* moe_last_error_string(void);

/* Number of kernels this library has launched (or recorded into a CUDA graph being
 * captured) in this process so far; a diagnostic for benchmarks. */
unsigned long long moe_launch_count(void);

/* Diagnostics: when dev_buffer is non-NULL, the fused decode kernel records per-CTA
 * timestamps (%globaltimer, 64 unsigned 64-bit slots per CTA, one row per CTA) into it; NULL
 * turns recording off. The buffer must hold 64 * (number of SMs) slots. */
void moe_debug_set_decode_trace(void* dev_buffer);

/* Testing aid for failure detection (process-wide; for tests only). `cycles` > 0 sets the limit,
 * in SM clock cycles, of the bounded waits of the single-token decode kernel (0 restores the
 * default of about two seconds). `extra_arrivals` > 0 makes that kernel's exchange between CTAs
 * wait for that many arrivals more than it launches: the wait cannot be satisfied, runs out, the
 * kernel records MOE_ERR_TIMEOUT in the workspace status word and exits without writing its
 * outputs. 0 turns it off. */
void moe_debug_set_wait_limit(unsigned long long cycles, int extra_arrivals);

/* Bytes of packed codes of one N x K matrix (N*K/2) and number of its bf16 scales
 * (N*K/128). Return 0 when N or K is not a positive multiple of 128. */
size_t moe_packed_bytes(int N, int K);
size_t moe_scales_count(int N, int K);

/* Symmetric group-128 int4 quantisation and packing of E matrices (abstract: "symmetric
 * group-128 four-bit weight quantization only to routed experts"). For each row n and group
 * of 128 consecutive K values w (bf16, read exactly as fp32):
 *   s = bf16_rne(max|w| / 7)   (fp32 IEEE division)
 *   q = clamp(rint(w / float(s)), -8, 7)   (fp32 IEEE division, round half to even;
 *                                           q = 0 where s == 0)
 * w_bf16: [E][N][K]; packed: [E][moe_packed_bytes(N,K)]; scales: [E][moe_scales_count(N,K)]
 * in the layout above. Errors: MOE_ERR_ARG (null/E<1), MOE_ERR_SHAPE (N or K % 128). */
int moe_quantize_pack(const uint16_t* w_bf16, int E, int N, int K,
                      uint8_t* packed, uint16_t* scales, moe_stream_t stream);

/* Top-k router (abstract: router kept in BF16, "unchanged top-k routing procedure").
 * logits: bf16 [T][E]. For each token: experts ordered by (logit descending, id ascending),
 * bf16 values compared exactly (-0 == +0); the first k are chosen. Softmax over all E in fp32,
 * the k chosen probabilities renormalised to sum to 1.
 * idx: int32 [T][k]; wts: fp32 [T][k]. Logits must be finite.
 * Errors: MOE_ERR_ARG (null, T < 0, k < 1, k > E), MOE_ERR_SHAPE (E > 256). */
int moe_route_topk(const uint16_t* logits_bf16, int T, int E, int k,
                   int32_t* idx, float* wts, moe_stream_t stream);

/* Groups the T*k (token, choice) pairs by expert ("fused grouped" execution).
 * counts[E]; offsets[E+1] exclusive prefix; perm[T*k]: pair id t*k+j of the p-th pair in
 * (expert, token, choice) order; inv[T*k]: position of pair t*k+j. idx values must be in
 * [0, E). scratch: int32 [moe_permute_scratch_count(T, k, E)]. */
size_t moe_permute_scratch_count(int T, int k, int E);
int moe_permute(const int32_t* idx, int T, int k, int E,
                int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv,
                int32_t* scratch, moe_stream_t stream);

/* Workspace of moe_w4a16_ffn / moe_w4a16_layer for these sizes (device memory, 256-byte
 * aligned, owned by the caller). It must be zeroed once with moe_workspace_init before its
 * first use; the kernels leave their counters zeroed again when they finish. A workspace sized
 * for T tokens serves calls with any T' <= T (any path) on the same H, I and E: the words that
 * must start at zero sit at offsets that depend on H, I and E only. Zero it again with
 * moe_workspace_init when H, I or E change, and after moe_workspace_status has reported a
 * failure. One workspace must not be used by two calls that can run at the same time. */
int moe_workspace_bytes(int T, int H, int I, int E, int k, size_t* bytes);
int moe_workspace_init(void* workspace, size_t bytes, moe_stream_t stream);

/* Reads (synchronously, on `stream`) and clears the workspace's device status word: 0 when
 * every kernel since the last read finished normally, else the MOE_ERR_* code of the first
 * failure (MOE_ERR_TIMEOUT: a bounded device-side wait ran out). */
int moe_workspace_status(void* workspace, moe_stream_t stream, int* status);

/* The W4A16 MoE FFN for routed tokens (abstract: "executes all selected experts through a
 * configurable GPU-resident slot cache and fused grouped MoE kernels"):
 *   y_e(x) = W2_e . ( silu(W_gate_e . x) * (W_up_e . x) ),  silu(z) = z / (1 + exp(-z))
 *   out[t] = sum_{j<k} wts[t][j] * y_{idx[t][j]}(x_t)
 * with W = q * s dequantised from the packed banks. The grouped tcgen05 path multiplies bf16
 * operands (bf16(q * s), and h rounded to bf16) with fp32 accumulation and keeps each
 * token-expert pair's down projection in fp32 until the router-weighted combine (when it splits
 * K in two, both halves add into the zeroed row: the same sum in either order); the fused decode
 * kernels (T <= 16) multiply the codes exactly with x and h held as 16-bit fixed point per
 * 128-element group (8-feature blocks for h at T = 1; error <= max|group| / 65278), scales
 * applied in fp32. out is bf16.
 *   x: bf16 [T][H]; idx, wts: the router's outputs [T][k].
 *   w13/s13: packed W13 ([2I][H]) per slot, w2/s2: packed W2 ([H][I]) per slot;
 *     slot stride = moe_packed_bytes / moe_scales_count of the matrix.
 *   slot_of_expert: int32 [E] device table, expert -> slot; NULL = identity (slot e holds
 *     expert e). An entry of -1 skips that expert's pairs (a later slot-cache wave runs them).
 *   workspace: see moe_workspace_bytes. out: bf16 [T][H], or NULL to leave this call's sum in
 *     the workspace's fp32 accumulator (a non-final slot-cache wave).
 * flags: a MOE_PATH_* value, optionally | MOE_FLAG_ACCUMULATE. Without ACCUMULATE the
 * accumulator is not read: this call's sum replaces it (out NULL) or is the output. With
 * ACCUMULATE, the sums of earlier waves in the accumulator are added. The fp32 accumulator is
 * zeroed again after out is written with ACCUMULATE.
 * Errors: MOE_ERR_ARG, MOE_ERR_SHAPE, MOE_ERR_CUDA (launch failure). */
int moe_w4a16_ffn(const uint16_t* x_bf16, int T, int H, int I, int E, int k,
                  const int32_t* idx, const float* wts,
                  const uint8_t* w13, const uint16_t* s13,
                  const uint8_t* w2, const uint16_t* s2,
                  const int32_t* slot_of_expert,
                  void* workspace, size_t workspace_bytes,
                  uint16_t* out_bf16, int flags, moe_stream_t stream);

/* Router + FFN of one layer in one call: moe_route_topk on logits, then moe_w4a16_ffn (with
 * MOE_PATH_DECODE the routing, grouping, both projections and the combine are one launch).
 * idx/wts receive the routing. Same arguments and errors as the two calls it stands for. */
int moe_w4a16_layer(const uint16_t* x_bf16, const uint16_t* logits_bf16,
                    int T, int H, int I, int E, int k,
                    const uint8_t* w13, const uint16_t* s13,
                    const uint8_t* w2, const uint16_t* s2,
                    const int32_t* slot_of_expert,
                    int32_t* idx, float* wts,
                    void* workspace, size_t workspace_bytes,
                    uint16_t* out_bf16, int flags, moe_stream_t stream);

/* moe_w4a16_layer without a caller workspace (the pages have no counterpart: this is a library
 * convenience). For callers that cannot allocate device memory - a program linking this C
 * library directly under a device-memory budget fixed up front, or a hot loop where an
 * allocation would synchronise the device - the workspace is a fixed 16 MiB array that the
 * library keeps in device memory (enough for the fused decode path at up to 16 tokens on a
 * 2048-wide, 64-expert, top-8 layer). Arguments as moe_w4a16_layer, minus the workspace.
 *  - The first call on a device looks up the array's device address (with that device
 *    current); make that first call before any stream capture on the device.
 *  - Every call on a device shares the array: calls that can run at the same time (other
 *    streams, other host threads) race, so the caller must serialise them.
 *  - Each call clears, on `stream`, the parts that must start at zero (control block and the
 *    fused-decode counters). A device-side failure (a bounded wait that ran out) is kept in the
 *    array's status word until moe_noalloc_status reads it.
 *  - Nothing is allocated.
 * Errors: MOE_ERR_SHAPE when these sizes need more than the array holds (use moe_w4a16_layer
 * with a caller workspace), MOE_ERR_ARG for MOE_FLAG_ACCUMULATE (the fp32 accumulator would be
 * shared by every call) and the errors of moe_w4a16_layer. */
int moe_w4a16_layer_noalloc(const uint16_t* x_bf16, const uint16_t* logits_bf16,
                            int T, int H, int I, int E, int k,
                            const uint8_t* w13, const uint16_t* s13,
                            const uint8_t* w2, const uint16_t* s2,
                            const int32_t* slot_of_expert,
                            int32_t* idx, float* wts,
                            uint16_t* out_bf16, int flags, moe_stream_t stream);

/* Reads (synchronously, on `stream`) and clears the status word of the array that
 * moe_w4a16_layer_noalloc uses on the current device: 0 when every call since the last read
 * finished normally on the device, else the MOE_ERR_* code of the first failure. */
int moe_noalloc_status(moe_stream_t stream, int* status);

/* ---- BF16 comparison layer (abstract: the W4A16 decode is compared with the same model in
 * BF16). The same layer on UNQUANTISED experts, through the same grouped scheduler and tcgen05
 * GEMMs (the weights loaded by TMA straight into the MMA operand, no dequantisation):
 *   w13_bf16: bf16 [slots][2I][H] ([W_gate; W_up] rows, row-major), w2_bf16: bf16 [slots][H][I];
 *   16-byte aligned. Everything else as moe_w4a16_ffn / moe_w4a16_layer (same workspace);
 *   flags: MOE_PATH_AUTO or MOE_PATH_GROUPED, optionally | MOE_FLAG_ACCUMULATE. The per-pair down
 * projection stays fp32 until the combine, as on the W4A16 grouped path.
 * Errors: MOE_ERR_ARG, MOE_ERR_SHAPE (H not a multiple of 256, as on the grouped path),
 * MOE_ERR_CUDA. */
int moe_bf16_ffn(const uint16_t* x_bf16, int T, int H, int I, int E, int k,
                 const int32_t* idx, const float* wts,
                 const uint16_t* w13_bf16, const uint16_t* w2_bf16,
                 const int32_t* slot_of_expert,
                 void* workspace, size_t workspace_bytes,
                 uint16_t* out_bf16, int flags, moe_stream_t stream);
int moe_bf16_layer(const uint16_t* x_bf16, const uint16_t* logits_bf16,
                   int T, int H, int I, int E, int k,
                   const uint16_t* w13_bf16, const uint16_t* w2_bf16,
                   const int32_t* slot_of_expert,
                   int32_t* idx, float* wts,
                   void* workspace, size_t workspace_bytes,
                   uint16_t* out_bf16, int flags, moe_stream_t stream);

/* ---- GPU slot cache (abstract: "configurable GPU-resident slot cache", experts kept in
 * pinned host memory). One cache per layer: S device slots, each holding one expert's packed
 * W13, W2 and their scales; misses are copied from the pinned host bank with
 * cudaMemcpyAsync on a copy stream. Replacement policy (the pages give none): hits keep their
 * slot; misses in ascending expert id take the lowest free slot, else evict the least recently
 * used slot not needed by the current wave (ties: lowest slot). A routed set larger than S runs
 * in waves of at most S experts (wave 1 = all hits + the first misses).                    */
typedef struct moe_slot_cache moe_slot_cache;

/* bank_* are HOST pointers to pinned memory (cudaHostAlloc / torch pin_memory) holding all E
 * experts in expert order; pool_* are device pointers with room for S experts in slot order.
 * Both stay owned by the caller and must outlive the cache. The cache starts empty.
 * *out receives a host-allocated handle. Creating the cache makes no CUDA call (the events of
 * moe_slot_cache_layer are created on its first call). Errors: MOE_ERR_ARG, MOE_ERR_SHAPE. */
int moe_slot_cache_create(int E, int S, int H, int I,
                          const uint8_t* bank_w13, const uint16_t* bank_s13,
                          const uint8_t* bank_w2, const uint16_t* bank_s2,
                          uint8_t* pool_w13, uint16_t* pool_s13,
                          uint8_t* pool_w2, uint16_t* pool_s2,
                          moe_slot_cache** out);
void moe_slot_cache_destroy(moe_slot_cache* cache);

/* Plans and starts one wave. needed_mask (HOST, ceil(E/64) words, bit e = expert e still has
 * to run) is read and the wave's experts are cleared from it; loop until it is zero.
 * wave_table (HOST, int32 [E]) receives each wave expert's slot and -1 for every other
 * expert; misses (HOST, int32 [S]) and *n_misses receive the experts loaded, in load order.
 * The copies wait for `reuse_ok` (an event recorded after the last kernel that read the pool;
 * may be NULL) and are issued on copy_stream; `loaded` (may be NULL) is recorded on
 * copy_stream after them. A failed copy returns MOE_ERR_CUDA with nothing of the wave
 * committed: needed_mask, the LRU clock and times are unchanged and no table is written; the
 * slots this wave had already started to overwrite are marked free (their contents are no
 * longer the experts they held). */
int slot_table_update(moe_slot_cache* cache, uint64_t* needed_mask,
                      int32_t* wave_table, int32_t* misses, int* n_misses,
                      moe_stream_t copy_stream, moe_event_t reuse_ok, moe_event_t loaded);

/* slot_table_update with two more knobs: at most max_wave experts in the wave (0 = S; more
 * than S is MOE_ERR_ARG), and protect (HOST, uint8 [S], may be NULL): nonzero marks a slot that
 * this wave must not overwrite (a wave still reading it). The wave is then the first
 * min(max_wave, hits) hits plus misses up to max_wave, both in ascending id, and a miss evicts
 * the least recently used slot that is neither protected nor holding a needed expert (one
 * waiting for a later wave included). slot_table_update is max_wave = 0, protect = NULL. */
int slot_table_update_ex(moe_slot_cache* cache, uint64_t* needed_mask,
                         int32_t* wave_table, int32_t* misses, int* n_misses,
                         moe_stream_t copy_stream, moe_event_t reuse_ok, moe_event_t loaded,
                         int max_wave, const uint8_t* protect);

/* Testing aid for failure handling: the n-th next refill copy of this cache (0 = the next
 * one) reports failure as if cudaMemcpyAsync had returned an error; n = -1 turns it off. */
void moe_slot_cache_fail_copy_after(moe_slot_cache* cache, int n);

/* Testing aid for the replacement policy: with dry != 0, slot_table_update plans and commits
 * every wave as usual but issues no copy (bank and pool are never touched), so the policy runs
 * on a machine without a GPU; dry = 0 restores the copies. */
void moe_slot_cache_dry_run(moe_slot_cache* cache, int dry);

/* Host view of the cache state: slot_expert[S] (-1 free), last_used[S]; returns the clock. */
int64_t moe_slot_cache_state(const moe_slot_cache* cache, int32_t* slot_expert, int64_t* last_used);

/* Runs one whole slot-cache layer: routing (idx/wts on device), a device->host read of the
 * routed expert set (the one synchronisation of this path), then for every wave
 * slot_table_update_ex + the FFN restricted to that wave's experts, accumulating in fp32; the
 * last wave writes out. With S >= 2 a wave holds at most S/2 experts and protects the slots of
 * the wave before it, so its refills overlap that wave's FFN (they wait only for the wave two
 * back); with S = 1 every refill waits for the wave before. wave_tables: device int32
 * [E * (ceil(E/S)+1)] scratch for the per-wave tables (reused in turn). Returns the number of
 * waves in *n_waves and the misses in *n_loads. */
int moe_slot_cache_layer(moe_slot_cache* cache,
                         const uint16_t* x_bf16, const uint16_t* logits_bf16, int T, int k,
                         int32_t* idx, float* wts, int32_t* wave_tables,
                         void* workspace, size_t workspace_bytes, uint16_t* out_bf16,
                         int path, moe_stream_t stream, moe_stream_t copy_stream,
                         int* n_waves, int* n_loads);

#ifdef __cplusplus
}
#endif

#endif /* MOE_W4A16_H */
