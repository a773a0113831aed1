// Shared definitions of the W4A16 MoE kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <stddef.h>

#include "moe_w4a16.h"

#define MOE_API extern "C" __attribute__((visibility("default")))

namespace moe {

constexpr int kGroup = 128;        // quantisation group along K
constexpr int kRowBlock = 128;     // rows per kernel tile (N is a multiple of it)
constexpr int kTileBytes = 8192;   // codes of one 128 x 128 tile
constexpr int kRowGroup = 8;       // rows per packed chunk
constexpr int kChunkBytes = 512;   // codes of one chunk: 8 rows x 128 K
constexpr int kMaxExperts = 256;

// Packed layout "MW4T v2" of a matrix W[N][K] (see include/moe_w4a16.h): byte offset of the
// 512-byte chunk of row group R = n / 8 and K group g, and index of its first scale.
__host__ __device__ __forceinline__ size_t chunk_offset(int R, int g, int G) {
  return ((size_t)R * G + g) * kChunkBytes;
}
__host__ __device__ __forceinline__ size_t chunk_scale_index(int R, int g, int G) {
  return ((size_t)R * G + g) * kRowGroup;
}
// Inside a chunk: the 16-byte piece of quarter kq (32 K values) of row r8 (0..7).
__host__ __device__ __forceinline__ int piece_offset(int kq, int r8) { return kq * 128 + r8 * 16; }

// ---- host-side error reporting (thread-local text, see moe_last_error_string) ----
int fail(int code, const char* fmt, ...);
int check_cuda(cudaError_t e, const char* what);
void note_launch();
inline int check_launch(const char* what) {
  note_launch();
  return check_cuda(cudaGetLastError(), what);
}

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }
inline int ceil_div(int a, int b) { return (a + b - 1) / b; }

// ---- workspace layout (all offsets 256-byte aligned) ----
struct WsLayout {
  size_t status;        // int32 status word + control counters (4 KiB block)
  size_t ctr;           // fused-decode counters (zero between launches); size set by H, I, E only,
                        // so the offset is the same for every T
  size_t counts;        // int32 [E]
  size_t offsets;       // int32 [E+1]
  size_t perm;          // int32 [T*k]
  size_t inv;           // int32 [T*k]
  size_t perm_scratch;  // int32 permute scratch
  size_t tiles;         // int32 [E+1] tile prefix + misc
  size_t tile_list;     // int32 [2][tile_list_len] grouped-GEMM tile lists (gate/up, down)
  size_t tile_list_len;
  size_t xp;            // bf16 [T*k][H] gathered activations
  size_t hp;            // bf16 [T*k][I] SwiGLU intermediate
  size_t yp;            // fp32 [T*k][H] per-pair down projection (grouped and reference paths)
  size_t acc;           // fp32 [T][H] accumulator for slot-cache waves
  size_t seq;           // int32 [E][E] one-expert slot tables of the sequential path
  size_t dec;           // fused-decode scratch
  size_t total;
};
WsLayout ws_layout(int T, int H, int I, int E, int k);

// Control block at the start of the workspace (int32 words).
enum CtlWord {
  kCtlStatus = 0,       // first device-side failure code (0 = none)
  kCtlWhere = 1,        // which wait gave up (diagnostic)
  kCtlClaim = 16,       // persistent-kernel work claim counter
  kCtlDone = 17,        // persistent-kernel exit counter
  kCtlDecode = 64,      // first word of the fused-decode counters
  kCtlWords = 1024
};

// Tensor maps over a packed bank (slots x N x K, layout MW4T v2) whose box is one 128 x 128 tile:
// codes as (32-bit word of a 512-byte chunk, K group, row group over all slots) with box
// (128, 1, 16); scales as (row in the chunk, K group, row group over all slots) with box
// (8, 1, 16). The tile of row block rb, K group g in slot s is at (0, g, s * N/8 + 16 * rb) and
// lands in shared memory as 16 chunks of 512 bytes (codes) or 128 scales in row order.
int make_chunk_code_map(void* map, const void* base, int N, int K, int slots);
int make_chunk_scale_map(void* map, const void* base, int N, int K, int slots);

size_t permute_scratch_count(int T, int k, int E);
size_t decode_scratch_bytes(int T, int H, int I, int E, int k);
size_t decode_counter_bytes(int H, int I, int E);

// ---- launch helpers (defined in the .cu files) ----
int launch_quantize_pack(const uint16_t* w, int E, int N, int K, uint8_t* packed, uint16_t* scales,
                         cudaStream_t s);
int launch_route(const uint16_t* logits, int T, int E, int k, int32_t* idx, float* wts, cudaStream_t s);
int launch_permute(const int32_t* idx, int T, int k, int E, int32_t* counts, int32_t* offsets,
                   int32_t* perm, int32_t* inv, int32_t* scratch, cudaStream_t s);

struct FfnArgs {
  const uint16_t* x; int T, H, I, E, k;
  const int32_t* idx; const float* wts;
  const uint8_t* w13; const uint16_t* s13;
  const uint8_t* w2; const uint16_t* s2;
  const int32_t* slot;    // may be null (identity)
  char* ws; size_t ws_bytes;
  uint16_t* out;          // may be null with accumulate
  bool accumulate;
  const uint16_t* logits; // fused decode: route in-kernel when non-null
  int32_t* idx_out; float* wts_out;
  bool bf16_weights;      // w13 / w2 hold unquantised bf16 rows (grouped path only; no scales)
};
int ffn_simple(const FfnArgs& a, cudaStream_t s);
int ffn_sequential(const FfnArgs& a, cudaStream_t s);
int ffn_decode(const FfnArgs& a, cudaStream_t s);
bool ffn_decode_supported(const FfnArgs& a);
int ffn_grouped(const FfnArgs& a, cudaStream_t s);
bool ffn_grouped_supported(const FfnArgs& a);

// Gather + tile-plan + combine pieces shared by the multi-launch paths.
int launch_gather_rows(const uint16_t* x, const int32_t* perm, int Tk, int k, int H, uint16_t* xp,
                       cudaStream_t s);
int launch_combine(const FfnArgs& a, const WsLayout& L, cudaStream_t s);

// Launch with programmatic stream serialisation (PDL): the kernel may start while the previous
// one on the stream finishes; every kernel launched this way calls pdl_begin() first.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// ---- device helpers ----
// Start of a PDL-launched kernel: wait until the previous kernel's results are visible, then let
// the next kernel start launching (it waits for this one the same way).
__device__ __forceinline__ void pdl_begin() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ float bf16_bits_to_float(uint32_t b) { return __uint_as_float(b << 16); }

__device__ __forceinline__ int slot_of(const int32_t* table, int e) { return table ? table[e] : e; }

// Records the first device-side failure in the workspace status word.
__device__ __forceinline__ void report_status(int* ctl, int code, int where) {
  if (atomicCAS(ctl + kCtlStatus, 0, code) == 0) ctl[kCtlWhere] = where;
}

}  // namespace moe
