// Context-sharded decode: one sequence's chunks split by chunk id over several shards (each a
// cache of its own, usually one per GPU).  Phase 1 on every shard is the ordinary selection
// kernel, which also exports the shard's own top k as candidates (score, global id).  The
// kernels here run phase 2 on a shard, once the caller has gathered every shard's candidates:
//   shard_select_kernel   the k best of all candidates (descending score, ascending global id:
//                         the unsharded selection, since a chunk among the k best overall is
//                         among its own shard's k best), and the ones this shard holds
//   shard_scan_kernel     those as an explicit tile list for the chunk-attention kernel
//   combine_partial_kernel per unit: the shard's pieces and raw tail merged, the predictor's
//                         second layer applied, left unnormalised: (m_j, l_j, y_j) per head
// and the merge of the gathered shard records (merge_partials_kernel):
//   o_j = sum_s w_s y_{s,j} / sum_s w_s l_{s,j},  w_s = 2^(m_{s,j} - max_s m_{s,j}).
// The softmax over the union of the shards' tokens regrouped by shard ("OjaKV", section 3,
// the attention equations); the page that motivates sharding: "LowRAM Compresses KV Cache
// Asymmetrically", section "Why Peak Throughput Can Improve by 5x" (moving the KV cache,
// also between GPUs, bounds decode).
#include <climits>

#include "lowram_internal.cuh"
#include "reuse.cuh"

namespace lowram {
namespace {

__device__ __forceinline__ uint32_t order_key(float x) {
  const uint32_t u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ int lane_excl_scan(int v) {
  const int lane = threadIdx.x & 31;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  return x - v;
}

// One warp per unit u of the call.  Candidates: cs / ci [n_shards][n_layers][B][Hkv][k], each
// shard's ids ascending, shards in ascending chunk-offset order (so the gathered list of a
// unit is ascending in global id).  Lane l holds candidates l*NPL .. l*NPL + NPL - 1.
template <int NPL>
__global__ void __launch_bounds__(32)
shard_select_kernel(Geom g, CacheBuffers cb, Scratch sc, const float* __restrict__ cs,
                    const int32_t* __restrict__ ci, int n_shards, int offset, int32_t* __restrict__ sel_out) {
  const int u = blockIdx.x;
  const Unit un = unit_of(g, u);
  const int l = g.layer0 + un.li;
  const int grp = l / g.G;
  const int NG = g.L / g.G;
  const int lane = threadIdx.x;
  const size_t ui = (size_t)(un.li * g.B + un.b) * g.Hkv + un.hkv;   // the caller's unit index
  const size_t per_shard = (size_t)g.n_layers * g.B * g.Hkv * g.k;
  const int n = n_shards * g.k;
  uint32_t key[NPL];
  int id[NPL];
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    const int j = lane * NPL + i;
    if (j < n) {
      const size_t at = (size_t)(j / g.k) * per_shard + ui * g.k + (j % g.k);
      key[i] = order_key(cs[at]);
      id[i] = ci[at];
    } else {
      key[i] = 0u;
      id[i] = INT_MAX;
    }
  }
  // candidates must come in ascending global id (see above)
  bool ordered = true;
#pragma unroll
  for (int i = 0; i + 1 < NPL; ++i) ordered &= lane * NPL + i + 1 >= n || id[i] < id[i + 1];
  const int next_first = __shfl_down_sync(0xffffffffu, id[0], 1);
  if (lane < 31 && (lane + 1) * NPL < n) ordered &= id[NPL - 1] < next_first;
  if (!__all_sync(0xffffffffu, ordered) && lane == 0) atomicOr(sc.err, ERR_SELECT);

  // the k-th largest key T: the largest T with #{key >= T} >= k
  uint32_t T = 0;
#pragma unroll 1
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t trial = T | (1u << bit);
    int cnt = 0;
#pragma unroll
    for (int i = 0; i < NPL; ++i) cnt += key[i] >= trial ? 1 : 0;
    if (__reduce_add_sync(0xffffffffu, cnt) >= g.k) T = trial;
  }
  int gt = 0, eq = 0;
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    gt += key[i] > T ? 1 : 0;
    eq += key[i] == T ? 1 : 0;
  }
  const int need_eq = g.k - (int)__reduce_add_sync(0xffffffffu, gt);
  const int n_eq = (int)__reduce_add_sync(0xffffffffu, eq);
  uint32_t take = 0;
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    if (key[i] > T) take |= 1u << i;
  }
  if (n_eq == need_eq) {
#pragma unroll
    for (int i = 0; i < NPL; ++i)
      if (key[i] == T) take |= 1u << i;
  } else {
    // more candidates tie at T than places left: the lowest global ids among them (rare:
    // each tied candidate counts the tied ones with a lower id)
    int below[NPL];
#pragma unroll
    for (int i = 0; i < NPL; ++i) below[i] = 0;
#pragma unroll 1
    for (int src = 0; src < 32; ++src) {
#pragma unroll
      for (int i2 = 0; i2 < NPL; ++i2) {
        const uint32_t k2 = __shfl_sync(0xffffffffu, key[i2], src);
        const int id2 = __shfl_sync(0xffffffffu, id[i2], src);
#pragma unroll
        for (int i = 0; i < NPL; ++i) below[i] += (k2 == T && id2 < id[i]) ? 1 : 0;
      }
    }
#pragma unroll
    for (int i = 0; i < NPL; ++i)
      if (key[i] == T && below[i] < need_eq) take |= 1u << i;
  }
  // the global selection in ascending id, and the part of it this shard holds
  int pos = lane_excl_scan(__popc(take));
  int lpos = 0;
  uint32_t mine = 0;
#pragma unroll
  for (int i = 0; i < NPL; ++i)
    if ((take >> i) & 1u && id[i] >= offset && id[i] < offset + g.nC) mine |= 1u << i;
  lpos = lane_excl_scan(__popc(mine));
  const int16_t* slot = cb.slot ? cb.slot + (((size_t)un.b * NG + grp) * g.Hkv + un.hkv) * g.nCs : nullptr;
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    if (!((take >> i) & 1u)) continue;
    if (sel_out && pos < g.k) sel_out[ui * g.k + pos] = id[i];
    ++pos;
    if ((mine >> i) & 1u) {
      const int c = id[i] - offset;
      int sl = slot ? (int)slot[c] : c;
      if (sl < 0 || sl >= g.nL) {
        atomicOr(sc.err, ERR_SELECT);
        sl = 0;
      }
      sc.sel_slot[(size_t)u * g.k + lpos] = sl;
      sc.sel_id[(size_t)u * g.k + lpos] = c;
      ++lpos;
    }
  }
  const int n_mine = (int)__reduce_add_sync(0xffffffffu, __popc(mine));
  if (lane == 0) sc.unit_ntile[u] = n_mine;
}

// One CTA: tile_ptr = exclusive prefix of the units' tile counts, the tile list, the total.
constexpr int kScanThreads = 1024;
__global__ void __launch_bounds__(kScanThreads)
shard_scan_kernel(int U, int k, Scratch sc) {
  __shared__ int part[kScanThreads];
  const int tid = threadIdx.x;
  const int per = (U + kScanThreads - 1) / kScanThreads;
  const int u0 = min(U, tid * per), u1 = min(U, u0 + per);
  int sum = 0;
  for (int u = u0; u < u1; ++u) sum += sc.unit_ntile[u];
  part[tid] = sum;
  __syncthreads();
  for (int o = 1; o < kScanThreads; o <<= 1) {   // inclusive scan of the per-thread sums
    const int v = tid >= o ? part[tid - o] : 0;
    __syncthreads();
    part[tid] += v;
    __syncthreads();
  }
  int base = part[tid] - sum;
  for (int u = u0; u < u1; ++u) {
    sc.tile_ptr[u] = base;
    base += sc.unit_ntile[u];
  }
  if (tid == kScanThreads - 1) {
    sc.tile_ptr[U] = part[tid];
    *sc.tile_total = part[tid];
  }
  __syncthreads();   // the offsets above are visible to the whole block
  // the list itself: one warp per unit, one lane per tile (coalesced)
  const int warp = tid >> 5, lane = tid & 31;
  for (int u = warp; u < U; u += kScanThreads / 32) {
    const int b0 = sc.tile_ptr[u], cnt = sc.tile_ptr[u + 1] - b0;
    for (int i = lane; i < cnt; i += 32) {
      sc.tile_unit[b0 + i] = u;
      sc.tile_slot[b0 + i] = sc.sel_slot[(size_t)u * k + i];
    }
  }
}

// Per unit: the shard's pieces (chunk partial records of the CTAs that ran its tiles) and its
// raw tail merged per head, W2 applied to the merged hidden sums, not normalised.  Output row
// of query head j: [0] m_j (log2 units), [1] l_j, [2 + t] y_j[t].
template <typename T>
__global__ void __launch_bounds__(256)
combine_partial_kernel(Geom g, CacheBuffers cb, Scratch sc, float* __restrict__ partial) {
  extern __shared__ __align__(16) float sm[];
  const int u = blockIdx.x;
  const Unit un = unit_of(g, u);
  const int l = g.layer0 + un.li;
  const int tid = threadIdx.x;
  const long long total = *sc.tile_total;
  const int p0 = sc.tile_ptr[u], p1 = sc.tile_ptr[u + 1];
  int c0 = 0, nrec = 0;
  if (p1 > p0) {
    c0 = cta_of_tile(total, g.P, p0);
    nrec = cta_of_tile(total, g.P, p1 - 1) - c0 + 1;
  }
  float* accH = sm;                    // [g][h]
  float* accD = accH + g.g * g.h;      // [g][d]
  float* wts = accD + g.g * g.d;       // [nrec + 1][g] merge weights (last row: tail)
  float* hm = wts + (size_t)(nrec + 1) * g.g;   // [g] merged max
  float* hl = hm + g.g;                // [g] merged sum
  const float* trec = sc.tail_part + (size_t)u * g.tail_stride;
  for (int j = tid; j < g.g; j += blockDim.x) {
    float M = trec[j];
    for (int r = 0; r < nrec; ++r) M = fmaxf(M, sc.part[(size_t)(u + c0 + r) * g.rec_stride + j]);
    float L = 0.f;
    for (int r = 0; r < nrec; ++r) {
      const float* rec = sc.part + (size_t)(u + c0 + r) * g.rec_stride;
      const float w = rec[j] == -INFINITY ? 0.f : exp2f(rec[j] - M);
      wts[r * g.g + j] = w;
      L = fmaf(w, rec[g.g + j], L);
    }
    const float wt = trec[j] == -INFINITY ? 0.f : exp2f(trec[j] - M);
    wts[nrec * g.g + j] = wt;
    hm[j] = M;
    hl[j] = fmaf(wt, trec[g.g + j], L);
  }
  __syncthreads();
  for (int i = tid; i < g.g * g.h; i += blockDim.x) {
    const int j = i / g.h;
    float a = 0.f;
    for (int r = 0; r < nrec; ++r) a = fmaf(wts[r * g.g + j], sc.part[(size_t)(u + c0 + r) * g.rec_stride + 2 * g.g + i], a);
    accH[i] = a;
  }
  for (int i = tid; i < g.g * g.d; i += blockDim.x) {
    const int j = i / g.d;
    float a = wts[nrec * g.g + j] * trec[2 * g.g + i];
    for (int r = 0; r < nrec; ++r)
      a = fmaf(wts[r * g.g + j], sc.part[(size_t)(u + c0 + r) * g.rec_stride + 2 * g.g + g.g * g.h + i], a);
    accD[i] = a;
  }
  __syncthreads();
  const T* w2 = reinterpret_cast<const T*>(cb.w2) + ((size_t)l * g.Hkv + un.hkv) * g.d * g.h;
  const size_t row0 = ((size_t)(un.li * g.B + un.b) * g.Hq + (size_t)un.hkv * g.g);
  for (int i = tid; i < g.g * g.d; i += blockDim.x) {
    const int j = i / g.d, t = i % g.d;
    const T* wr = w2 + (size_t)t * g.h;
    const float* ah = accH + j * g.h;
    float a = 0.f;
    for (int e = 0; e < g.h; ++e) a = fmaf(to_f(wr[e]), ah[e], a);
    partial[(row0 + j) * (g.d + 2) + 2 + t] = a + accD[i];
  }
  for (int j = tid; j < g.g; j += blockDim.x) {
    partial[(row0 + j) * (g.d + 2)] = hm[j];
    partial[(row0 + j) * (g.d + 2) + 1] = hl[j];
  }
}

// One CTA per output row: the shards' records merged and normalised.
template <typename T>
__global__ void __launch_bounds__(256)
merge_partials_kernel(int n_parts, long long n_rows, int d, const float* __restrict__ parts, T* __restrict__ out) {
  const long long row = blockIdx.x;
  const size_t rs = (size_t)d + 2;
  float M = -INFINITY;
  for (int s = 0; s < n_parts; ++s) M = fmaxf(M, parts[((size_t)s * n_rows + row) * rs]);
  float den = 0.f;
  for (int s = 0; s < n_parts; ++s) {
    const float* p = parts + ((size_t)s * n_rows + row) * rs;
    den = fmaf(p[0] == -INFINITY ? 0.f : exp2f(p[0] - M), p[1], den);
  }
  for (int t = threadIdx.x; t < d; t += blockDim.x) {
    float num = 0.f;
    for (int s = 0; s < n_parts; ++s) {
      const float* p = parts + ((size_t)s * n_rows + row) * rs;
      num = fmaf(p[0] == -INFINITY ? 0.f : exp2f(p[0] - M), p[2 + t], num);
    }
    out[(size_t)row * d + t] = from_f<T>(num / den);
  }
}

}  // namespace

cudaError_t launch_shard_select(const Geom& g, const CacheBuffers& cb, const Scratch& sc, const float* cand_score,
                                const int32_t* cand_id, int n_shards, int offset, int32_t* sel_out, cudaStream_t s) {
  const int n = n_shards * g.k;
  if (n <= 64)
    shard_select_kernel<2><<<g.U, 32, 0, s>>>(g, cb, sc, cand_score, cand_id, n_shards, offset, sel_out);
  else if (n <= 256)
    shard_select_kernel<8><<<g.U, 32, 0, s>>>(g, cb, sc, cand_score, cand_id, n_shards, offset, sel_out);
  else if (n <= 1024)
    shard_select_kernel<32><<<g.U, 32, 0, s>>>(g, cb, sc, cand_score, cand_id, n_shards, offset, sel_out);
  else
    return cudaErrorInvalidValue;
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  shard_scan_kernel<<<1, kScanThreads, 0, s>>>(g.U, g.k, sc);
  return cudaGetLastError();
}

cudaError_t launch_tile_scan(const Geom& g, const Scratch& sc, cudaStream_t s) {
  shard_scan_kernel<<<1, kScanThreads, 0, s>>>(g.U, g.k, sc);
  return cudaGetLastError();
}

cudaError_t launch_combine_partial(const Geom& g, const CacheBuffers& cb, const Scratch& sc, int dtype,
                                   float* partial, cudaStream_t s) {
  // bf16, d = 128, h = 256, g in {4, 8}, k <= 32: the warp-MMA combine writes the partials
  if (dtype != LOWRAM_F32 && g.d == 128 && g.h == 256 && (g.g == 4 || g.g == 8) && g.k <= 32)
    return launch_combine_partial_fast(g, cb, sc, partial, s);
  const int max_pieces = g.k < g.P ? g.k : g.P;
  const size_t smem = sizeof(float) * ((size_t)g.g * g.h + (size_t)g.g * g.d + (size_t)(max_pieces + 1) * g.g + 2 * g.g);
  if (smem > 227 * 1024) return cudaErrorInvalidConfiguration;
  if (dtype == LOWRAM_F32) {
    auto k = combine_partial_kernel<float>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<g.U, 256, smem, s>>>(g, cb, sc, partial);
  } else {
    auto k = combine_partial_kernel<__nv_bfloat16>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<g.U, 256, smem, s>>>(g, cb, sc, partial);
  }
  return cudaGetLastError();
}

cudaError_t launch_merge_partials(int n_parts, long long n_rows, int d, const float* parts, int out_dtype, void* out,
                                  cudaStream_t s) {
  if (n_rows <= 0) return cudaSuccess;
  if (out_dtype == LOWRAM_F32)
    merge_partials_kernel<float><<<(unsigned)n_rows, 128, 0, s>>>(n_parts, n_rows, d, parts, static_cast<float*>(out));
  else
    merge_partials_kernel<__nv_bfloat16><<<(unsigned)n_rows, 128, 0, s>>>(n_parts, n_rows, d, parts,
                                                                          static_cast<__nv_bfloat16*>(out));
  return cudaGetLastError();
}

}  // namespace lowram
