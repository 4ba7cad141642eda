// Internal declarations of the rebuilt-chunk reuse store (reuse.cu; not part of the C ABI).
#pragma once

#include "lowram_internal.cuh"

namespace lowram {

// Device view of a reuse store (the C ABI's lowram_reuse holds the allocations).
struct ReuseDev {
  __nv_bfloat16* entries;        // [E][C][d]: rebuilt values of one (unit, chunk) each
  int32_t* table;                // [B][L][Hkv][table_stride]: entry of each chunk slot, or -1
  long long* owner;              // [E]: table index an entry serves, or -1
  int32_t* ring;                 // [2]: next entry to fill; [1] its copy taken by the plan kernel
  unsigned long long* counters;  // [3]: hits, misses, fills (cumulative)
  int32_t* hit_entry;            // [U][k] per call: the unit's hit entries ...
  int32_t* hit_slot;             // [U][k] ... and their chunk slots
  int32_t* hit_n;                // [U]
  float* hit_part;               // [U][tail_stride]: the hits' softmax record (tail format)
  const __half* w2h;             // [L][Hkv][d][h]: W2 in fp16 for the fill kernel's MMA
  int E, fill_cap;
  long long table_stride;
};

bool reuse_supported(const Geom& g, int dtype, int store);
// bf16 -> fp16 copy of n elements (encode.cu).
cudaError_t launch_to_half(const __nv_bfloat16* src, __half* dst, size_t n, cudaStream_t s);
// phase 0: plan (hits / misses) and the misses' tile list; 1: attention over the hits;
// 2: fills of the first fill_cap misses and the table update.
cudaError_t launch_reuse(const Geom& g, const CacheBuffers& cb, const Scratch& sc, const ReuseDev& st,
                         const void* w1f_tc, int n_sm, cudaStream_t s, int phase);
// The tile list of the selections in sc.sel_slot / sc.unit_ntile (shard.cu).
cudaError_t launch_tile_scan(const Geom& g, const Scratch& sc, cudaStream_t s);
// Combine over an explicit tile list plus one extra record per unit in the tail's format
// (the reuse store's hits), normalised (combine.cu).
// Per unit the pieces of the tile list and the tail merged, W2 applied, left unnormalised:
// rows [m (log2 units), l, y[0..d)] per (layer, sequence, query head) (a context shard's
// partial), on the warp-MMA combine (bf16, d = 128, h = 256, g in {4, 8}, k <= 32); combine.cu.
cudaError_t launch_combine_partial_fast(const Geom& g, const CacheBuffers& cb, const Scratch& sc, float* partial,
                                        cudaStream_t s);
cudaError_t launch_combine_list(const Geom& g, const CacheBuffers& cb, const Scratch& sc, const float* extra_rec,
                                void* out, cudaStream_t s);

}  // namespace lowram
