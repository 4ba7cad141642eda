// Internal declarations of the decode-loop upkeep of a cache (repack.cu): tail append,
// residual-record re-layout and tail shift after a re-pack.  Not part of the C ABI.
#pragma once

#include "lowram_internal.cuh"

namespace lowram {

// Error-word bit of the upkeep kernels (next to the ERR_* bits of lowram_internal.cuh).
constexpr uint32_t ERR_TAIL_FULL = 1u << 6;   // an append found a full tail: token dropped

// The error word inside an encoder workspace (encode.cu): bounded-wait timeouts of the
// encoder's tensor-core kernels.
uint32_t* encode_error_word(const Geom& g, void* workspace, bool folds_given = false);

// launch_encode with the folds a cache already holds: w1f_t the fp32 W1' = W1 B_l^T
// [L][Hkv][r][h], w1f_tc its bf16 halves [L][Hkv][h][r] (native stores; unused for int8),
// so the encoder does not fold again; w2h_ready: the workspace already holds the fp16 copy
// of W2 from an earlier call with the same weights.
cudaError_t launch_encode(const Geom& g, int store, int n_res, const void* keys, const void* values,
                          const void* basis, const void* w1, const void* w2, const lowram_encode_dst& dst,
                          void* workspace, cudaStream_t s, const float* w1f_t, const void* w1f_tc,
                          bool w2h_ready);

// A re-pack that cannot write the new chunk in place re-lays the cache with room for this
// many more chunks per unit (and as many records per unit as this re-pack keeps per chunk):
// max(kSpareChunksMin, live chunks / kSpareChunksDiv).
constexpr int kSpareChunksMin = 4;
constexpr int kSpareChunksDiv = 16;

// row_bytes: bytes of one tail row / record row, a multiple of 16.  Strides: res_ptr rows of
// nLs + 1 entries, slot rows of nCs entries.
cudaError_t launch_append(int B, int L, int Hkv, int T, int row_bytes, const void* k_new, const void* v_new,
                          void* tail_k, void* tail_v, int32_t* tail_len, uint32_t* err, cudaStream_t s);
// *flag != 0 afterwards if some unit lacks room for n_res records after its last chunk's.
cudaError_t launch_repack_room(int U, int nL, int nLs, int n_res, const int32_t* res_ptr, long long n_records,
                               uint32_t* flag, cudaStream_t s);
cudaError_t launch_repack_scan(int U, int nL, int nLs, long long spare_rec, const int32_t* old_ptr,
                               const int32_t* new_ptr, long long* base, uint32_t* err, cudaStream_t s);
cudaError_t launch_repack_records(int U, int nL, int nLs_old, int nLs_new, int row_bytes, long long n_old,
                                  long long n_new_total, const int32_t* old_ptr, const uint16_t* old_pos,
                                  const void* old_val, const __half* old_scale, const int32_t* new_ptr,
                                  const uint16_t* new_pos, const void* new_val, const __half* new_scale,
                                  const long long* base, int32_t* out_ptr, uint16_t* out_pos, void* out_val,
                                  __half* out_scale, uint32_t* err, cudaStream_t s);
cudaError_t launch_repack_append_records(int U, int nL, int nLs, int row_bytes, long long n_records,
                                         long long n_new_total, const int32_t* new_ptr, const uint16_t* new_pos,
                                         const void* new_val, const __half* new_scale, int32_t* res_ptr,
                                         uint16_t* res_pos, void* res_val, __half* res_scale, uint32_t* err,
                                         cudaStream_t s);
cudaError_t launch_repack_slot(long long rows, int nCs, int nC, int nL, int16_t* slot, cudaStream_t s);
cudaError_t launch_tail_shift(int B, int L, int Hkv, int T, int C, int row_bytes, void* tail_k, void* tail_v,
                              int32_t* tail_len, cudaStream_t s);

}  // namespace lowram
