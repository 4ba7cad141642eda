// Upkeep of the cache in a decode loop: append each step's keys and values to the raw tail,
// and re-pack the tail's oldest chunk into the compressed store.
//
// Tokens generated after prefill stay uncompressed in the tail (rit.work "lowram-kv-cache-
// compression", section on values and keys: generated tokens are kept raw).  Once every
// tail holds at least C tokens, the oldest C of every (sequence, layer, KV head) are
// encoded with the given basis and predictor ("LowRAM Compresses KV Cache Asymmetrically",
// "Cross-Layer Low-Rank Key Compression" and "Core Mechanism") by the encoder kernels into
// one new chunk; the kernels here move the rest: the residual records re-laid in unit order
// with the new chunk's records after each unit's old ones, and the tail shifted down by C.
// All of them are copies and index arithmetic: bound by HBM.
#include "upkeep.cuh"

namespace lowram {
namespace {

constexpr int kCopyThreads = 256;

// One warp per (layer, sequence, KV head) row of the step's keys / values
// [L][B][Hkv][d]: 16-byte pieces into tail slot tail_len[b].
__global__ void __launch_bounds__(kCopyThreads)
append_rows_kernel(int B, int L, int Hkv, int T, int row16, const uint4* __restrict__ k_new,
                   const uint4* __restrict__ v_new, uint4* __restrict__ tail_k, uint4* __restrict__ tail_v,
                   const int32_t* __restrict__ tail_len, uint32_t* __restrict__ err) {
  const int lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * (kCopyThreads / 32) + (threadIdx.x >> 5);
  if (row >= (long long)L * B * Hkv) return;
  const int h = (int)(row % Hkv);
  const int b = (int)((row / Hkv) % B);
  const int l = (int)(row / ((long long)Hkv * B));
  const int t = tail_len[b];
  if (t < 0 || t >= T) {
    if (lane == 0) atomicOr(err, t < 0 ? ERR_TAIL_LEN : ERR_TAIL_FULL);
    return;
  }
  const size_t dst = ((((size_t)b * L + l) * Hkv + h) * T + t) * row16;
  for (int i = lane; i < row16; i += 32) {
    tail_k[dst + i] = k_new[row * row16 + i];
    tail_v[dst + i] = v_new[row * row16 + i];
  }
}

// tail_len[b] += 1 where the rows were written (after append_rows_kernel).
__global__ void append_count_kernel(int B, int T, int32_t* __restrict__ tail_len) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < B && tail_len[b] >= 0 && tail_len[b] < T) tail_len[b] += 1;
}

// Record bases of the re-laid cache: unit u (order (b, l, KV head)) gets its old records
// [old_ptr[u][0], old_ptr[u][nL]), its new chunk's [new_ptr[u][0], new_ptr[u][1]) and
// spare_rec spare rows; base[u] is the exclusive prefix sum of those counts, base[U] the
// total.  old_ptr rows have nLs + 1 entries.  One block.
__global__ void __launch_bounds__(1024)
repack_scan_kernel(int U, int nL, int nLs, long long spare_rec, const int32_t* __restrict__ old_ptr,
                   const int32_t* __restrict__ new_ptr, long long* __restrict__ base, uint32_t* __restrict__ err) {
  __shared__ long long part[1024];
  const int tid = threadIdx.x;
  const int per = (U + blockDim.x - 1) / blockDim.x;
  const int u0 = min(U, tid * per), u1 = min(U, u0 + per);
  auto count = [&](int u) -> long long {
    const int32_t* op = old_ptr + (size_t)u * (nLs + 1);
    const long long o = (long long)op[nL] - op[0];
    const long long n = (long long)new_ptr[2 * (size_t)u + 1] - new_ptr[2 * (size_t)u];
    if (o < 0 || n < 0) {
      atomicOr(err, ERR_RES_PTR);
      return spare_rec;
    }
    return o + n + spare_rec;
  };
  long long s = 0;
  for (int u = u0; u < u1; ++u) s += count(u);
  part[tid] = s;
  __syncthreads();
  for (int off = 1; off < (int)blockDim.x; off <<= 1) {   // inclusive scan (Hillis-Steele)
    const long long v = tid >= off ? part[tid - off] : 0;
    __syncthreads();
    part[tid] += v;
    __syncthreads();
  }
  long long run = part[tid] - s;
  for (int u = u0; u < u1; ++u) {
    base[u] = run;
    run += count(u);
  }
  if (tid == blockDim.x - 1) base[U] = part[tid];
}

// Room check of an in-place re-pack: unit u's records end before the next unit's region
// starts (the array's end for the last unit), so n_res more fit after them.
__global__ void repack_room_kernel(int U, int nL, int nLs, int n_res, const int32_t* __restrict__ res_ptr,
                                   long long n_records, uint32_t* __restrict__ flag) {
  const int u = blockIdx.x * blockDim.x + threadIdx.x;
  if (u >= U) return;
  const long long start = res_ptr[(size_t)u * (nLs + 1) + nL];
  const long long end = u + 1 < U ? (long long)res_ptr[(size_t)(u + 1) * (nLs + 1)] : n_records;
  if (start < 0 || start + n_res > end) atomicOr(flag, 1u);
}

// One CTA per unit: its old records, then its new chunk's, to base[u] onwards; the first
// nL + 2 offsets of the unit's CSR row (rows of nLs_new + 1).  Record rows are row16 pieces
// of 16 bytes.
__global__ void __launch_bounds__(kCopyThreads)
repack_records_kernel(int nL, int nLs_old, int nLs_new, int row16, long long n_old, long long n_new_total,
                      const int32_t* __restrict__ old_ptr, const uint16_t* __restrict__ old_pos,
                      const uint4* __restrict__ old_val, const __half* __restrict__ old_scale,
                      const int32_t* __restrict__ new_ptr, const uint16_t* __restrict__ new_pos,
                      const uint4* __restrict__ new_val, const __half* __restrict__ new_scale,
                      const long long* __restrict__ base, int32_t* __restrict__ out_ptr,
                      uint16_t* __restrict__ out_pos, uint4* __restrict__ out_val,
                      __half* __restrict__ out_scale, uint32_t* __restrict__ err) {
  const int u = blockIdx.x;
  const int32_t* op = old_ptr + (size_t)u * (nLs_old + 1);
  const long long o0 = op[0], no = (long long)op[nL] - o0;
  const long long e0 = new_ptr[2 * (size_t)u], ne = (long long)new_ptr[2 * (size_t)u + 1] - e0;
  const long long b0 = base[u];
  const bool ok_old = no >= 0 && o0 >= 0 && o0 + no <= n_old;
  const bool ok_new = ne >= 0 && e0 >= 0 && e0 + ne <= n_new_total;
  if ((!ok_old || !ok_new) && threadIdx.x == 0) atomicOr(err, ERR_RES_PTR);
  int32_t* orow = out_ptr + (size_t)u * (nLs_new + 1);
  for (int c = threadIdx.x; c <= nL; c += blockDim.x) orow[c] = (int32_t)(b0 + (ok_old ? op[c] - o0 : 0));
  if (threadIdx.x == 0) orow[nL + 1] = (int32_t)(b0 + (ok_old ? no : 0) + (ok_new ? ne : 0));
  if (ok_old) {
    for (long long i = threadIdx.x; i < no * row16; i += blockDim.x)
      out_val[(b0 * row16) + i] = old_val[o0 * row16 + i];
    for (long long i = threadIdx.x; i < no; i += blockDim.x) {
      out_pos[b0 + i] = old_pos[o0 + i];
      if (out_scale) out_scale[b0 + i] = old_scale[o0 + i];
    }
  }
  if (ok_new) {
    const long long d0 = b0 + (ok_old ? no : 0);
    for (long long i = threadIdx.x; i < ne * row16; i += blockDim.x)
      out_val[(d0 * row16) + i] = new_val[e0 * row16 + i];
    for (long long i = threadIdx.x; i < ne; i += blockDim.x) {
      out_pos[d0 + i] = new_pos[e0 + i];
      if (out_scale) out_scale[d0 + i] = new_scale[e0 + i];
    }
  }
}

// In-place re-pack, one CTA per unit: the new chunk's records go right after the unit's
// last ones (the room check has passed) and the unit's CSR row gains offset nL + 1.
__global__ void __launch_bounds__(kCopyThreads)
repack_append_records_kernel(int nL, int nLs, int row16, long long n_records, long long n_new_total,
                             const int32_t* __restrict__ new_ptr, const uint16_t* __restrict__ new_pos,
                             const uint4* __restrict__ new_val, const __half* __restrict__ new_scale,
                             int32_t* __restrict__ res_ptr, uint16_t* __restrict__ res_pos,
                             uint4* __restrict__ res_val, __half* __restrict__ res_scale, uint32_t* __restrict__ err) {
  const int u = blockIdx.x;
  int32_t* row = res_ptr + (size_t)u * (nLs + 1);
  const long long d0 = row[nL];
  const long long e0 = new_ptr[2 * (size_t)u], ne = (long long)new_ptr[2 * (size_t)u + 1] - e0;
  if (ne < 0 || e0 < 0 || e0 + ne > n_new_total || d0 < 0 || d0 + ne > n_records) {
    if (threadIdx.x == 0) atomicOr(err, ERR_RES_PTR);
    return;
  }
  for (long long i = threadIdx.x; i < ne * row16; i += blockDim.x) res_val[d0 * row16 + i] = new_val[e0 * row16 + i];
  for (long long i = threadIdx.x; i < ne; i += blockDim.x) {
    res_pos[d0 + i] = new_pos[e0 + i];
    if (res_scale) res_scale[d0 + i] = new_scale[e0 + i];
  }
  if (threadIdx.x == 0) row[nL + 1] = (int32_t)(d0 + ne);
}

// The new chunk's slot under eviction: entry nC of every slot row (rows of nCs) is nL.
__global__ void repack_slot_kernel(long long rows, int nCs, int nC, int nL, int16_t* __restrict__ slot) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < rows) slot[i * nCs + nC] = (int16_t)nL;
}

// One CTA per (b, l, KV head): tail rows [C, len) move to [0, len - C), a block of C rows at
// a time (a block's source and destination are disjoint, and a block only overwrites rows
// earlier blocks have already read).
__global__ void __launch_bounds__(kCopyThreads)
tail_shift_kernel(int L, int Hkv, int T, int C, int row16, uint4* __restrict__ tail_k, uint4* __restrict__ tail_v,
                  const int32_t* __restrict__ tail_len) {
  const int u = blockIdx.x;                         // (b * L + l) * Hkv + h
  const int b = u / (L * Hkv);
  const int n = min(tail_len[b], T) - C;
  uint4* tk = tail_k + (size_t)u * T * row16;
  uint4* tv = tail_v + (size_t)u * T * row16;
  for (int j0 = 0; j0 < n; j0 += C) {
    const int rows = min(C, n - j0);
    for (int i = threadIdx.x; i < rows * row16; i += blockDim.x) {
      const size_t dst = (size_t)j0 * row16 + i;
      tk[dst] = tk[dst + (size_t)C * row16];
      tv[dst] = tv[dst + (size_t)C * row16];
    }
    __syncthreads();
  }
}

__global__ void tail_drop_kernel(int B, int C, int32_t* __restrict__ tail_len) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < B) tail_len[b] -= C;
}

}  // namespace

cudaError_t launch_append(int B, int L, int Hkv, int T, int row_bytes, const void* k_new, const void* v_new,
                          void* tail_k, void* tail_v, int32_t* tail_len, uint32_t* err, cudaStream_t s) {
  const long long rows = (long long)L * B * Hkv;
  const int per = kCopyThreads / 32;
  append_rows_kernel<<<(unsigned)((rows + per - 1) / per), kCopyThreads, 0, s>>>(
      B, L, Hkv, T, row_bytes / 16, static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new),
      static_cast<uint4*>(tail_k), static_cast<uint4*>(tail_v), tail_len, err);
  append_count_kernel<<<(B + 255) / 256, 256, 0, s>>>(B, T, tail_len);
  return cudaGetLastError();
}

cudaError_t launch_repack_room(int U, int nL, int nLs, int n_res, const int32_t* res_ptr, long long n_records,
                               uint32_t* flag, cudaStream_t s) {
  repack_room_kernel<<<(U + 255) / 256, 256, 0, s>>>(U, nL, nLs, n_res, res_ptr, n_records, flag);
  return cudaGetLastError();
}

cudaError_t launch_repack_scan(int U, int nL, int nLs, long long spare_rec, const int32_t* old_ptr,
                               const int32_t* new_ptr, long long* base, uint32_t* err, cudaStream_t s) {
  repack_scan_kernel<<<1, 1024, 0, s>>>(U, nL, nLs, spare_rec, old_ptr, new_ptr, base, err);
  return cudaGetLastError();
}

cudaError_t launch_repack_records(int U, int nL, int nLs_old, int nLs_new, int row_bytes, long long n_old,
                                  long long n_new_total, const int32_t* old_ptr, const uint16_t* old_pos,
                                  const void* old_val, const __half* old_scale, const int32_t* new_ptr,
                                  const uint16_t* new_pos, const void* new_val, const __half* new_scale,
                                  const long long* base, int32_t* out_ptr, uint16_t* out_pos, void* out_val,
                                  __half* out_scale, uint32_t* err, cudaStream_t s) {
  repack_records_kernel<<<U, kCopyThreads, 0, s>>>(
      nL, nLs_old, nLs_new, row_bytes / 16, n_old, n_new_total, old_ptr, old_pos, static_cast<const uint4*>(old_val),
      old_scale, new_ptr, new_pos, static_cast<const uint4*>(new_val), new_scale, base, out_ptr, out_pos,
      static_cast<uint4*>(out_val), out_scale, err);
  return cudaGetLastError();
}

cudaError_t launch_repack_append_records(int U, int nL, int nLs, int row_bytes, long long n_records,
                                         long long n_new_total, const int32_t* new_ptr, const uint16_t* new_pos,
                                         const void* new_val, const __half* new_scale, int32_t* res_ptr,
                                         uint16_t* res_pos, void* res_val, __half* res_scale, uint32_t* err,
                                         cudaStream_t s) {
  repack_append_records_kernel<<<U, kCopyThreads, 0, s>>>(
      nL, nLs, row_bytes / 16, n_records, n_new_total, new_ptr, new_pos, static_cast<const uint4*>(new_val),
      new_scale, res_ptr, res_pos, static_cast<uint4*>(res_val), res_scale, err);
  return cudaGetLastError();
}

cudaError_t launch_repack_slot(long long rows, int nCs, int nC, int nL, int16_t* slot, cudaStream_t s) {
  repack_slot_kernel<<<(unsigned)((rows + 255) / 256), 256, 0, s>>>(rows, nCs, nC, nL, slot);
  return cudaGetLastError();
}

cudaError_t launch_tail_shift(int B, int L, int Hkv, int T, int C, int row_bytes, void* tail_k, void* tail_v,
                              int32_t* tail_len, cudaStream_t s) {
  tail_shift_kernel<<<(unsigned)((long long)B * L * Hkv), kCopyThreads, 0, s>>>(
      L, Hkv, T, C, row_bytes / 16, static_cast<uint4*>(tail_k), static_cast<uint4*>(tail_v), tail_len);
  tail_drop_kernel<<<(B + 255) / 256, 256, 0, s>>>(B, C, tail_len);
  return cudaGetLastError();
}

}  // namespace lowram
