// Internal declarations of the LowRAM decode library (not part of the C ABI).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "lowram.h"

namespace lowram {

// Error-word bits written by device-side checks (never a trap).
enum : uint32_t {
  ERR_SLOT = 1u << 0,       // slot map not a compaction of live chunks
  ERR_RES_PTR = 1u << 1,    // CSR offsets decreasing or out of range
  ERR_RES_POS = 1u << 2,    // record position >= C or not increasing
  ERR_TAIL_LEN = 1u << 3,   // tail_len outside [0, T]
  ERR_TIMEOUT = 1u << 4,    // a bounded wait in a kernel ran out
  ERR_SELECT = 1u << 5,     // a selected chunk was evicted (cannot happen with valid tables)
};

constexpr int kMaxG = 16;          // query heads per KV head
constexpr int kMaxD = 256;         // head dim
constexpr int kMaxR = 512;         // rank
constexpr int kMaxH = 1024;        // predictor hidden width
constexpr int kMaxChunks = 8192;   // chunks per unit
constexpr int kMaxTail = 4096;
constexpr int kResPad = 32;        // zero rows kept after a cache's residual rows

// Geometry shared by every kernel of one decode call.
struct Geom {
  int B, L, G, Hkv, Hq, g, d, r, h, N, C, nC, nL, k, T;
  int nLs, nCs;        // per-unit strides of the chunk arrays: live slots (coefficient rows /
                       // C, summaries, CSR offsets - 1) and chunk ids (slot map); >= nL, nC
  int layer0, n_layers;
  int U;               // units in this call: n_layers * Hkv * B
  int P;               // CTAs of the chunk-attention kernel (tile partition)
  int rec_stride;      // floats per chunk partial record
  int tail_stride;     // floats per tail partial record
  int max_rec;         // upper bound of chunk records per unit (CTAs a unit's tiles touch)
  float qk_scale_log2; // log2(e) / sqrt(d)
  long long wait_cycles;  // limit of the tensor-core kernel's main-loop waits (SM cycles)
};

// Default limit of a bounded wait inside a kernel: about one second of SM clock.
constexpr long long kDefaultWaitCycles = 2000000000LL;

// Unit u enumerates (layer, KV head, sequence) with the sequence fastest, so the units
// that share one layer's weights are adjacent.
struct Unit {
  int li, hkv, b;
};
__host__ __device__ inline Unit unit_of(const Geom& g, int u) {
  Unit x;
  x.b = u % g.B;
  int t = u / g.B;
  x.hkv = t % g.Hkv;
  x.li = t / g.Hkv;
  return x;
}

// Tiles (unit, i-th selected chunk) are split over P CTAs in contiguous ranges;
// CTA c owns tiles [tile_begin(c), tile_begin(c+1)).  The partial record of the piece
// (unit u, CTA c) is record u + c.  With fewer tiles than CTAs (an explicit tile list is
// counted on the device, after the grid is sized) CTA c takes tile c alone and the empty
// CTAs are the last ones, so the CTAs holding one unit's tiles are consecutive and every one
// of them writes that unit's record.
__host__ __device__ inline long long tile_begin(long long total, int P, int c) {
  if (total < P) return c < total ? c : total;
  return (total * (long long)c) / P;
}
// Every CTA owns at least floor(total/P) >= 1 tiles, so the k tiles of one unit touch at
// most ceil((k-1)/floor(total/P)) + 1 CTAs.
__host__ __device__ inline int max_records_per_unit(long long total, int P, int k) {
  const long long minsize = total / P > 0 ? total / P : 1;
  int m = (int)((k - 1) / minsize) + 2;
  return m > k + 1 ? k + 1 : m;
}
// The CTA whose range holds tile x.
__host__ __device__ inline int cta_of_tile(long long total, int P, long long x) {
  if (total < P) return (int)x;
  // largest c with floor(c*total/P) <= x  <=>  c = ceil((x+1)*P/total) - 1
  long long num = (x + 1) * (long long)P;
  return (int)((num + total - 1) / total) - 1;
}

struct CacheBuffers {
  const void* coeff;
  const __half* coeff_scale;
  const void* basis;
  const void* w1;
  const void* w2;
  const void* summary;
  const int16_t* slot;
  const int32_t* res_ptr;
  const uint16_t* res_pos;
  const void* res_val;
  const __half* res_scale;
  const void* tail_k;
  const void* tail_v;
  const int32_t* tail_len;
  int64_t n_records;
};

struct Scratch {
  float* qt;          // [U][g][r] fp32: (B_l q_j) * log2(e)/sqrt(d)
  void* qt_tc;        // [U][16][r] 16-bit copy of qt for the tensor-core path (rows >= g zero)
  int32_t* sel_slot;  // [U][k] storage slot of each selected chunk (ids ascending)
  int32_t* sel_id;    // [U][k] chunk ids
  float* part;        // chunk partial records
  float* tail_part;   // [U][tail_stride]
  uint32_t* err;      // device error word
  // Explicit tile list (context-sharded decode; tile_total == nullptr otherwise): tile x of
  // the call is chunk slot tile_slot[x] of unit tile_unit[x], units in ascending order; unit
  // u's tiles are [tile_ptr[u], tile_ptr[u + 1]); *tile_total tiles in all.
  int32_t* tile_unit;
  int32_t* tile_slot;
  int32_t* tile_ptr;
  int32_t* tile_total;
  int32_t* unit_ntile; // [U] tiles of each unit (written by the shard selection)
};

// ---------------------------------------------------------------- element conversions

template <typename T> __device__ __forceinline__ float to_f(T x);
template <> __device__ __forceinline__ float to_f<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}
template <> __device__ __forceinline__ float to_f<__half>(__half x) { return __half2float(x); }
template <> __device__ __forceinline__ float to_f<int8_t>(int8_t x) { return (float)x; }

template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}
template <> __device__ __forceinline__ __half from_f<__half>(float x) { return __float2half_rn(x); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// ----------------------------------------------------------------------- launchers

// Optional output of the selection for context-sharded decode: the selected chunks' scores
// and ids + offset (the shard's first global chunk id), [n_layers][B][Hkv][k] like sel.
struct SelCand {
  float* score;
  int32_t* id;
  int offset;
};

// Steps 1-2 (+ the raw tail's partial softmax): one CTA per unit.
// tc_q_mode: 0 = no 16-bit copy of qt, 1 = bf16 copy, 2 = fp16 copy.
cudaError_t launch_select(const Geom& g, const CacheBuffers& cb, const Scratch& sc,
                          int dtype, const void* q, float* scores_out, int32_t* sel_out,
                          int tc_q_mode, bool tail, cudaStream_t s, SelCand cand = SelCand{nullptr, nullptr, 0});
// Steps 3-5 on CUDA cores over the selected chunks.  w1f_t holds the fp32 W1' of layers
// [w1f_layer0, ...): layer l's fold is at (l - w1f_layer0) * Hkv * r * h.
cudaError_t launch_attend_simt(const Geom& g, const CacheBuffers& cb, const Scratch& sc,
                               int dtype, int store, const float* w1f_t, int w1f_layer0,
                               cudaStream_t s);
// Steps 3-5 on tcgen05 tensor cores.  Returns cudaErrorNotSupported for shapes it
// does not handle.
cudaError_t launch_attend_tc(const Geom& g, const CacheBuffers& cb, const Scratch& sc,
                             int store, const void* w1f_tc, int n_sm, cudaStream_t s);
bool attend_tc_supported(const Geom& g, int dtype, int store);
// Split merge, second predictor layer and normalisation.
cudaError_t launch_combine(const Geom& g, const CacheBuffers& cb, const Scratch& sc,
                           int dtype, void* out, cudaStream_t s);
// Create-time fold W1' = W1 . B_l^T (fp32 transposed [r][h] for CUDA cores; 16-bit
// [h][r] scaled by 1/2 for tensor cores).
cudaError_t launch_fold(const Geom& g, const CacheBuffers& cb, int dtype, int store,
                        float* w1f_t, void* w1f_tc, cudaStream_t s);
// Prefill-side encoder (dense K, V -> compressed arrays); bf16, d = 128, h = 256,
// r in {64, 128}, C in {64, 128}.  The workspace holds the fp32 W1' fold, the residual
// norms and the flags; with folds_given (the caller passes both W1' folds, as the re-pack
// does) the fold regions are left out.
size_t encode_workspace_bytes(const Geom& g, bool folds_given = false);
cudaError_t launch_encode(const Geom& g, int store, int n_res, const void* keys, const void* values,
                          const void* basis, const void* w1, const void* w2, const lowram_encode_dst& dst,
                          void* workspace, cudaStream_t s);
// Context-sharded decode, phase 2 (shard.cu): the global selection from every shard's
// candidates and the shard's tile list (sc.tile_*), the shard's unnormalised partial per query
// head ([n_layers][B][Hq][d + 2]: m in log2 units, l, y), and the merge of the shards' partials.
cudaError_t launch_shard_select(const Geom& g, const CacheBuffers& cb, const Scratch& sc, const float* cand_score,
                                const int32_t* cand_id, int n_shards, int offset, int32_t* sel_out, cudaStream_t s);
cudaError_t launch_combine_partial(const Geom& g, const CacheBuffers& cb, const Scratch& sc, int dtype,
                                   float* partial, cudaStream_t s);
cudaError_t launch_merge_partials(int n_parts, long long n_rows, int d, const float* parts, int out_dtype, void* out,
                                  cudaStream_t s);
// Device-side table checks.
cudaError_t launch_validate(const Geom& g, const CacheBuffers& cb, uint32_t* err,
                            cudaStream_t s);

}  // namespace lowram
