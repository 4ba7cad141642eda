// Final step: merge the softmax partials of a unit (raw tail + every chunk piece),
// apply the predictor's second layer once to the softmax-weighted hidden sum and
// normalise:
//     o_j = (W2 . sum_t p_jt h_t + sum_t p_jt delta_t + sum_tail p_jt v_t) / sum_t p_jt
// This is the exact regrouping of sum_t p_jt (W2 h_t + delta_t) for the rebuilt values of
// "LowRAM Compresses KV Cache Asymmetrically", section "Core Mechanism" (Vhat = f(K) plus
// delta for the worst tokens), inside the attention of "OjaKV", section 3.
// Also: the create-time fold W1' = W1 B_l^T and the device-side table check.
#include "lowram_internal.cuh"

namespace lowram {
namespace {

constexpr int kThreads = 256;

// 8 consecutive row elements as floats (one 16-byte load for bf16, two for fp32).
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&v)[8]) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}
__device__ __forceinline__ void load8(const float* p, float (&v)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

template <typename T>
__global__ void __launch_bounds__(kThreads)
combine_kernel(Geom g, CacheBuffers cb, Scratch sc, T* __restrict__ out) {
  extern __shared__ __align__(16) float sm[];
  const int u = blockIdx.x;
  const Unit un = unit_of(g, u);
  const int l = g.layer0 + un.li;
  const long long total = (long long)g.U * g.k;
  const int c0 = cta_of_tile(total, g.P, (long long)u * g.k);
  const int c1 = cta_of_tile(total, g.P, (long long)(u + 1) * g.k - 1);
  const int nrec = c1 - c0 + 1;
  if (nrec > g.max_rec) {  // cannot happen with a consistent tile partition
    if (threadIdx.x == 0) atomicOr(sc.err, ERR_SELECT);
    return;
  }
  const int tid = threadIdx.x;

  float* accH = sm;                   // [g][h]
  float* accD = accH + g.g * g.h;     // [g][d]
  float* lsum = accD + g.g * g.d;     // [g]
  float* wts = lsum + g.g;            // [nrec + 1][g]  (last row: tail)

  const float* trec = sc.tail_part + (size_t)u * g.tail_stride;
  for (int j = tid; j < g.g; j += blockDim.x) {
    float M = trec[j];
    for (int r = 0; r < nrec; ++r) M = fmaxf(M, sc.part[(size_t)(u + c0 + r) * g.rec_stride + j]);
    float L = 0.f;
    for (int r = 0; r < nrec; ++r) {
      const float* rec = sc.part + (size_t)(u + c0 + r) * g.rec_stride;
      const float w = rec[j] == -INFINITY ? 0.f : exp2f(rec[j] - M);
      wts[r * g.g + j] = w;
      L += w * rec[g.g + j];
    }
    const float wt = trec[j] == -INFINITY ? 0.f : exp2f(trec[j] - M);
    wts[nrec * g.g + j] = wt;
    L += wt * trec[g.g + j];
    lsum[j] = L;
  }
  __syncthreads();
  for (int i = tid; i < g.g * g.h; i += blockDim.x) {
    const int j = i / g.h;
    float a = 0.f;
    for (int r = 0; r < nrec; ++r)
      a = fmaf(wts[r * g.g + j], sc.part[(size_t)(u + c0 + r) * g.rec_stride + 2 * g.g + i], a);
    accH[i] = a;
  }
  for (int i = tid; i < g.g * g.d; i += blockDim.x) {
    const int j = i / g.d;
    float a = wts[nrec * g.g + j] * trec[2 * g.g + i];
    for (int r = 0; r < nrec; ++r)
      a = fmaf(wts[r * g.g + j],
               sc.part[(size_t)(u + c0 + r) * g.rec_stride + 2 * g.g + g.g * g.h + i], a);
    accD[i] = a;
  }
  __syncthreads();
  // second predictor layer on the weighted hidden sums: one thread per (output row dd,
  // group of up to 4 heads), W2 rows read with 16-byte loads, accH broadcast from smem
  const T* W2 = reinterpret_cast<const T*>(cb.w2) + ((size_t)l * g.Hkv + un.hkv) * g.d * g.h;
  T* o = out + ((size_t)(un.li * g.B + un.b) * g.Hq + (size_t)un.hkv * g.g) * g.d;
  const int jgroups = (g.g + 3) / 4;
  for (int item = tid; item < g.d * jgroups; item += blockDim.x) {
    const int dd = item % g.d, j0 = (item / g.d) * 4;
    const T* row = W2 + (size_t)dd * g.h;
    float a[4] = {0.f, 0.f, 0.f, 0.f};
    if ((g.h & 7) == 0) {
      for (int i = 0; i < g.h; i += 8) {
        float v[8];
        load8(row + i, v);
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          if (j0 + jj < g.g) {
            const float* hsum = accH + (j0 + jj) * g.h + i;
#pragma unroll
            for (int x = 0; x < 8; ++x) a[jj] = fmaf(v[x], hsum[x], a[jj]);
          }
        }
      }
    } else {
      for (int i = 0; i < g.h; ++i) {
        const float v = to_f(row[i]);
#pragma unroll
        for (int jj = 0; jj < 4; ++jj)
          if (j0 + jj < g.g) a[jj] = fmaf(v, accH[(j0 + jj) * g.h + i], a[jj]);
      }
    }
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      const int j = j0 + jj;
      if (j < g.g) o[(size_t)j * g.d + dd] = from_f<T>((a[jj] + accD[j * g.d + dd]) / lsum[j]);
    }
  }
}

// The same merge for bf16 with d = 128, h = 256, g in {4, 8}, arranged as one round trip to
// memory: every thread issues all its loads on entry -- its half of one W2 row (16 x 16
// bytes) and, for each of its float4 slices of the weighted sums, the slice of every piece
// record with that head's running max and sum -- then derives the merge weights of its
// head itself (max over the pieces, 2^(m_r - M)), so the only barrier is the one before
// the second predictor layer reads the merged hidden sums.  Up to kFastRec pieces per unit
// (a unit's k chunk tiles touch at most two CTAs at the bench sizes; more take the generic kernel).
constexpr int kFastRec = 2;

template <int GQ>
__global__ void __launch_bounds__(kThreads, 2)
combine_fast_kernel(Geom g, CacheBuffers cb, Scratch sc, __nv_bfloat16* __restrict__ out) {
  constexpr int D = 128, H = 256;
  constexpr int NH = GQ * H / 4 / kThreads;          // float4 slices of the hidden sums per thread
  constexpr int ND = (GQ * D / 4 + kThreads - 1) / kThreads;
  extern __shared__ __align__(16) float sm[];
  const int u = blockIdx.x;
  const Unit un = unit_of(g, u);
  const int l = g.layer0 + un.li;
  const int tid = threadIdx.x;
  // this thread's half of W2 row dd, requested before anything else
  const int dd = tid >> 1, half = tid & 1;
  const uint4* wrow = reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(cb.w2) +
                                                     (((size_t)l * g.Hkv + un.hkv) * D + dd) * H + half * (H / 2));
  uint4 w[H / 16];
#pragma unroll
  for (int e = 0; e < H / 16; ++e) w[e] = __ldg(wrow + e);

  const long long total = (long long)g.U * g.k;
  const int c0 = cta_of_tile(total, g.P, (long long)u * g.k);
  const int c1 = cta_of_tile(total, g.P, (long long)(u + 1) * g.k - 1);
  const int nrec = c1 - c0 + 1;
  if (nrec > g.max_rec || nrec > kFastRec) {  // cannot happen with a consistent tile partition
    if (tid == 0) atomicOr(sc.err, ERR_SELECT);
    return;
  }
  float* accH = sm;                 // [GQ][H]
  float* accD = accH + GQ * H;      // [GQ][D]
  float* lsum = accD + GQ * D;      // [GQ]
  const float* trec = sc.tail_part + (size_t)u * g.tail_stride;
  const float* rec0 = sc.part + (size_t)(u + c0) * g.rec_stride;
  // merge weights of head j over the pieces (and the tail): w_r = 2^(m_r - M)
  auto weights = [&](int j, const float (&m)[kFastRec], float mt, float (&wr)[kFastRec], float& wt) {
    float M = mt;
#pragma unroll
    for (int r = 0; r < kFastRec; ++r)
      if (r < nrec) M = fmaxf(M, m[r]);
#pragma unroll
    for (int r = 0; r < kFastRec; ++r) wr[r] = (r < nrec && m[r] != -INFINITY) ? exp2f(m[r] - M) : 0.f;
    wt = mt == -INFINITY ? 0.f : exp2f(mt - M);
  };
  // hidden sums: loads first
  float4 vh[NH][kFastRec];
  float mh[NH][kFastRec];
#pragma unroll
  for (int q = 0; q < NH; ++q) {
    const int i4 = tid + q * kThreads, j = (i4 * 4) / H;
#pragma unroll
    for (int r = 0; r < kFastRec; ++r) {
      const float* rec = rec0 + (size_t)r * g.rec_stride;
      if (r < nrec) {
        mh[q][r] = rec[j];
        vh[q][r] = *reinterpret_cast<const float4*>(rec + 2 * GQ + i4 * 4);
      }
    }
  }
  // residual / tail sums: loads first
  float4 vd[ND][kFastRec], vt[ND];
  float md[ND][kFastRec], mtd[ND];
#pragma unroll
  for (int q = 0; q < ND; ++q) {
    const int i4 = tid + q * kThreads;
    if (i4 < GQ * D / 4) {
      const int j = (i4 * 4) / D;
      mtd[q] = trec[j];
      vt[q] = *reinterpret_cast<const float4*>(trec + 2 * GQ + i4 * 4);
#pragma unroll
      for (int r = 0; r < kFastRec; ++r) {
        const float* rec = rec0 + (size_t)r * g.rec_stride;
        if (r < nrec) {
          md[q][r] = rec[j];
          vd[q][r] = *reinterpret_cast<const float4*>(rec + 2 * GQ + GQ * H + i4 * 4);
        }
      }
    }
  }
  // the softmax denominators
  if (tid < GQ) {
    const int j = tid;
    float m[kFastRec], sr[kFastRec], wr[kFastRec], wt;
#pragma unroll
    for (int r = 0; r < kFastRec; ++r) {
      const float* rec = rec0 + (size_t)r * g.rec_stride;
      m[r] = r < nrec ? rec[j] : -INFINITY;
      sr[r] = r < nrec ? rec[GQ + j] : 0.f;
    }
    const float mt = trec[j], st = trec[GQ + j];
    weights(j, m, mt, wr, wt);
    float L = wt * st;
#pragma unroll
    for (int r = 0; r < kFastRec; ++r) L = fmaf(wr[r], sr[r], L);
    lsum[j] = L;
  }
#pragma unroll
  for (int q = 0; q < NH; ++q) {
    const int i4 = tid + q * kThreads, j = (i4 * 4) / H;
    float wr[kFastRec], wt;
    weights(j, mh[q], trec[j], wr, wt);
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int r = 0; r < kFastRec; ++r) {
      if (r < nrec) {
        a.x = fmaf(wr[r], vh[q][r].x, a.x); a.y = fmaf(wr[r], vh[q][r].y, a.y);
        a.z = fmaf(wr[r], vh[q][r].z, a.z); a.w = fmaf(wr[r], vh[q][r].w, a.w);
      }
    }
    *reinterpret_cast<float4*>(accH + i4 * 4) = a;
  }
#pragma unroll
  for (int q = 0; q < ND; ++q) {
    const int i4 = tid + q * kThreads;
    if (i4 < GQ * D / 4) {
      const int j = (i4 * 4) / D;
      float wr[kFastRec], wt;
      weights(j, md[q], mtd[q], wr, wt);
      float4 a = make_float4(wt * vt[q].x, wt * vt[q].y, wt * vt[q].z, wt * vt[q].w);
#pragma unroll
      for (int r = 0; r < kFastRec; ++r) {
        if (r < nrec) {
          a.x = fmaf(wr[r], vd[q][r].x, a.x); a.y = fmaf(wr[r], vd[q][r].y, a.y);
          a.z = fmaf(wr[r], vd[q][r].z, a.z); a.w = fmaf(wr[r], vd[q][r].w, a.w);
        }
      }
      *reinterpret_cast<float4*>(accD + i4 * 4) = a;
    }
  }
  __syncthreads();
  // second predictor layer: this thread's half row against every head's hidden sums
  float a[GQ];
#pragma unroll
  for (int j = 0; j < GQ; ++j) a[j] = 0.f;
#pragma unroll
  for (int e = 0; e < H / 16; ++e) {
    const uint32_t ww[4] = {w[e].x, w[e].y, w[e].z, w[e].w};
#pragma unroll
    for (int h2 = 0; h2 < 4; ++h2) {
      const float v0 = __uint_as_float(ww[h2] << 16), v1 = __uint_as_float(ww[h2] & 0xffff0000u);
      const int m = half * (H / 2) + e * 8 + 2 * h2;
#pragma unroll
      for (int j = 0; j < GQ; ++j) a[j] = fmaf(v1, accH[j * H + m + 1], fmaf(v0, accH[j * H + m], a[j]));
    }
  }
#pragma unroll
  for (int j = 0; j < GQ; ++j) a[j] += __shfl_xor_sync(0xffffffffu, a[j], 1);
  if (half == 0) {
    __nv_bfloat16* o = out + ((size_t)(un.li * g.B + un.b) * g.Hq + (size_t)un.hkv * GQ) * D;
#pragma unroll
    for (int j = 0; j < GQ; ++j) o[(size_t)j * D + dd] = __float2bfloat16_rn((a[j] + accD[j * D + dd]) / lsum[j]);
  }
}

// W1'[i][rr] = sum_dd W1[i][dd] * B_l[rr][dd] for every (layer, KV head).  A block computes a
// 32 (hidden) x 64 (rank) tile of one (layer, KV head) with both operands staged through
// shared memory 32 columns of d at a time; thread (ty, tx) accumulates hidden rows 2ty, 2ty+1
// and ranks 4tx .. 4tx+3.
template <typename T>
__global__ void __launch_bounds__(256)
fold_tiled_kernel(Geom g, const T* __restrict__ w1, const T* __restrict__ basis, float* __restrict__ w1f_t,
                  __nv_bfloat16* __restrict__ w1f_bf16, __half* __restrict__ w1f_f16) {
  constexpr int TI = 32, TR = 64, TK = 32;
  __shared__ float ws[TI][TK + 1];
  __shared__ float bs[TR][TK + 1];
  const int i0 = blockIdx.x * TI, r0 = blockIdx.y * TR;
  const size_t lh = blockIdx.z;
  const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
  float acc[2][4] = {};
  for (int k0 = 0; k0 < g.d; k0 += TK) {
    for (int p = tid; p < TI * TK; p += 256) {
      const int i = p / TK, k = p % TK;
      ws[i][k] = (i0 + i < g.h && k0 + k < g.d) ? to_f(w1[(lh * g.h + i0 + i) * g.d + k0 + k]) : 0.f;
    }
    for (int p = tid; p < TR * TK; p += 256) {
      const int rr = p / TK, k = p % TK;
      bs[rr][k] = (r0 + rr < g.r && k0 + k < g.d) ? to_f(basis[(lh * g.r + r0 + rr) * g.d + k0 + k]) : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int k = 0; k < TK; ++k) {
      const float a0 = ws[2 * ty][k], a1 = ws[2 * ty + 1][k];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float bv = bs[4 * tx + j][k];
        acc[0][j] = fmaf(a0, bv, acc[0][j]);
        acc[1][j] = fmaf(a1, bv, acc[1][j]);
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int ii = 0; ii < 2; ++ii) {
    const int i = i0 + 2 * ty + ii;
    if (i >= g.h) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int rr = r0 + 4 * tx + j;
      if (rr >= g.r) continue;
      const float a = acc[ii][j];
      if (w1f_t) w1f_t[(lh * g.r + rr) * g.h + i] = a;
      // tensor-core copy holds W1'/2: the MMA then yields u = x/2 and silu(x) = u + u*tanh(u)
      if (w1f_bf16) w1f_bf16[(lh * g.h + i) * g.r + rr] = __float2bfloat16_rn(0.5f * a);
      if (w1f_f16) w1f_f16[(lh * g.h + i) * g.r + rr] = __float2half_rn(0.5f * a);
    }
  }
}

__global__ void validate_kernel(Geom g, CacheBuffers cb, uint32_t* err) {
  const int NG = g.L / g.G;
  const int n_slot_rows = g.B * NG * g.Hkv;
  const int n_units = g.B * g.L * g.Hkv;
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx < n_slot_rows && cb.slot) {
    const int16_t* s = cb.slot + (size_t)idx * g.nCs;
    int next = 0;
    bool bad = false;
    for (int c = 0; c < g.nC; ++c) {
      const int v = s[c];
      if (v == -1) continue;
      if (v != next) bad = true;
      ++next;
    }
    if (next != g.nL) bad = true;
    if (bad) atomicOr(err, ERR_SLOT);
  }
  if (idx < n_units) {
    const int32_t* p = cb.res_ptr + (size_t)idx * (g.nLs + 1);
    bool bad_ptr = false, bad_pos = false;
    for (int s = 0; s <= g.nL; ++s) {
      if (p[s] < 0 || p[s] > cb.n_records) bad_ptr = true;
      if (s < g.nL && p[s + 1] < p[s]) bad_ptr = true;
    }
    if (!bad_ptr) {
      for (int s = 0; s < g.nL; ++s) {
        int prev = -1;
        for (int r = p[s]; r < p[s + 1]; ++r) {
          const int pos = cb.res_pos[r];
          if (pos >= g.C || pos <= prev) bad_pos = true;
          prev = pos;
        }
      }
    }
    if (bad_ptr) atomicOr(err, ERR_RES_PTR);
    if (bad_pos) atomicOr(err, ERR_RES_POS);
  }
  if (idx < g.B) {
    const int tl = cb.tail_len[idx];
    if (tl < 0 || tl > g.T) atomicOr(err, ERR_TAIL_LEN);
  }
}

}  // namespace

size_t combine_smem_bytes(const Geom& g) {
  return sizeof(float) * ((size_t)g.g * g.h + (size_t)g.g * g.d + g.g + (size_t)(g.max_rec + 1) * g.g);
}

cudaError_t launch_combine(const Geom& g, const CacheBuffers& cb, const Scratch& sc, int dtype,
                           void* out, cudaStream_t s) {
  const size_t smem = combine_smem_bytes(g);
  if (smem > 227 * 1024) return cudaErrorInvalidConfiguration;
  cudaError_t e;
  if (dtype == LOWRAM_F32) {
    auto k = combine_kernel<float>;
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<g.U, kThreads, smem, s>>>(g, cb, sc, static_cast<float*>(out));
  } else if (g.d == 128 && g.h == 256 && (g.g == 4 || g.g == 8) && g.max_rec <= kFastRec) {
    auto k = g.g == 4 ? combine_fast_kernel<4> : combine_fast_kernel<8>;
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<g.U, kThreads, smem, s>>>(g, cb, sc, static_cast<__nv_bfloat16*>(out));
  } else {
    auto k = combine_kernel<__nv_bfloat16>;
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<g.U, kThreads, smem, s>>>(g, cb, sc, static_cast<__nv_bfloat16*>(out));
  }
  return cudaGetLastError();
}

cudaError_t launch_fold(const Geom& g, const CacheBuffers& cb, int dtype, int store,
                        float* w1f_t, void* w1f_tc, cudaStream_t s) {
  const dim3 grid((g.h + 31) / 32, (g.r + 63) / 64, g.L * g.Hkv);
  if (dtype == LOWRAM_F32) {
    fold_tiled_kernel<float><<<grid, 256, 0, s>>>(g, static_cast<const float*>(cb.w1),
                                                  static_cast<const float*>(cb.basis), w1f_t, nullptr, nullptr);
  } else {
    __nv_bfloat16* bf = store == LOWRAM_STORE_INT8 ? nullptr : static_cast<__nv_bfloat16*>(w1f_tc);
    __half* hf = store == LOWRAM_STORE_INT8 ? static_cast<__half*>(w1f_tc) : nullptr;
    fold_tiled_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(
        g, static_cast<const __nv_bfloat16*>(cb.w1), static_cast<const __nv_bfloat16*>(cb.basis), w1f_t, bf, hf);
  }
  return cudaGetLastError();
}

cudaError_t launch_validate(const Geom& g, const CacheBuffers& cb, uint32_t* err, cudaStream_t s) {
  const int n = g.B * g.L * g.Hkv;
  validate_kernel<<<(n + 127) / 128, 128, 0, s>>>(g, cb, err);
  return cudaGetLastError();
}

}  // namespace lowram
