// Steps 1-2 of decode-time attention over a LowRAM-compressed KV cache: chunk scores
// against the step's queries and the top-k chunk selection, plus the raw tail's partial
// softmax.  One CTA per unit (sequence, layer, KV head).
//
// Chunk score (the pages fix no summary or score; this library's reading): the chunk's
// mean rebuilt key at layer l is abar_c . B_l, so
//     s_c = sum_j q_j . (abar_c B_l) / sqrt(d) = (B_l sum_j q_j) . abar_c / sqrt(d),
// computed in the coefficient space ("OjaKV", section 3.1: queries projected into the key
// basis).  Selection: "LowRAM: Low-Rank Keys and Amortised Values ..." abstract (only a
// selected subset is reconstructed per step); rit.work "lowram-kv-cache-compression",
// section "Значения предсказывают, ключи раскладывают по общему базису" (fragments chosen
// by the current query; new tokens kept uncompressed).  Ties go to the lower chunk id.
//
// Work is spread so that no thread waits on a chain of shuffles: every projection, score
// and tail logit is one thread's dot product over 16-byte loads; top-k of up to 1024 chunks
// is a rank count over the keys in shared memory (bitonic sort above that).
#include "lowram_internal.cuh"

namespace lowram {
namespace {

constexpr int kThreads = 256;
constexpr int kTailBlock = 256;
constexpr int kRankMax = 1024;   // rank-count top-k up to this many chunks

__device__ __forceinline__ uint32_t float_order(float x) {
  uint32_t u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__host__ __device__ __forceinline__ int next_pow2(int n) {
  int p = 1;
  while (p < n) p <<= 1;
  return p;
}

// Bitonic sort, ascending, of n (power of two) 64-bit keys in shared memory.
__device__ void bitonic_sort(unsigned long long* keys, int n) {
  for (int size = 2; size <= n; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = threadIdx.x; i < (n >> 1); i += blockDim.x) {
        int lo = (i / stride) * stride * 2 + (i % stride);
        int hi = lo + stride;
        bool up = (lo & size) == 0;
        unsigned long long a = keys[lo], b = keys[hi];
        if ((a > b) == up) {
          keys[lo] = b;
          keys[hi] = a;
        }
      }
      __syncthreads();
    }
  }
}

// 8 consecutive elements of a row as floats (16-byte load for bf16, two for fp32).
template <typename T> struct Vec8;
template <> struct Vec8<__nv_bfloat16> {
  static __device__ __forceinline__ void load(const __nv_bfloat16* p, float (&v)[8]) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
};
template <> struct Vec8<float> {
  static __device__ __forceinline__ void load(const float* p, float (&v)[8]) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(p));
    const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
};

// dot(row[0:n], x[0:n]) with x in shared memory; n % 8 == 0 uses vector loads.
template <typename T>
__device__ __forceinline__ float row_dot(const T* row, const float* x, int n) {
  float a = 0.f;
  if ((n & 7) == 0) {
    for (int e = 0; e < n; e += 8) {
      float v[8];
      Vec8<T>::load(row + e, v);
#pragma unroll
      for (int i = 0; i < 8; ++i) a = fmaf(v[i], x[e + i], a);
    }
  } else {
    for (int e = 0; e < n; ++e) a = fmaf(to_f(row[e]), x[e], a);
  }
  return a;
}

template <typename T>
__global__ void __launch_bounds__(kThreads)
select_kernel(Geom g, CacheBuffers cb, Scratch sc, const T* __restrict__ q,
              float* __restrict__ scores_out, int32_t* __restrict__ sel_out, int tc_q_mode,
              int do_tail) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int u = blockIdx.x;
  const Unit un = unit_of(g, u);
  const int l = g.layer0 + un.li;
  const int grp = l / g.G;
  const int NG = g.L / g.G;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarp = blockDim.x >> 5;
  const bool rank_topk = g.nC <= kRankMax;
  const int nCp = rank_topk ? g.nC : next_pow2(g.nC);
  const int kp = next_pow2(g.k);

  unsigned long long* keys = reinterpret_cast<unsigned long long*>(smem_raw);  // [nCp]
  float* qs = reinterpret_cast<float*>(keys + nCp);                             // [g][d]
  float* qt = qs + g.g * g.d;                                                   // [g][r]
  float* qsum = qt + g.g * g.r;                                                 // [r]
  float* sc_s = qsum + g.r;                                                     // [nC]
  int* selv = reinterpret_cast<int*>(sc_s + g.nC);                              // [max(kp, nC)]
  float* lg = reinterpret_cast<float*>(selv + max(kp, g.nC));                   // [g][kTailBlock]
  float* acc = lg + g.g * kTailBlock;                                           // [g][d]
  float* mrun = acc + g.g * g.d;                                                // [g]
  float* lrun = mrun + g.g;                                                     // [g]
  float* alpha = lrun + g.g;                                                    // [g]

  // --- the unit's queries
  const size_t qoff = ((size_t)(un.li * g.B + un.b) * g.Hq + (size_t)un.hkv * g.g) * g.d;
  for (int i = tid; i < g.g * g.d; i += blockDim.x) qs[i] = to_f(q[qoff + i]);
  __syncthreads();

  // --- qt_j = B_l q_j: one thread per (basis row, group of up to 4 heads)
  const T* Bl = reinterpret_cast<const T*>(cb.basis) + ((size_t)l * g.Hkv + un.hkv) * g.r * g.d;
  const int jgroups = (g.g + 3) / 4;
  for (int item = tid; item < g.r * jgroups; item += blockDim.x) {
    const int i = item % g.r, j0 = (item / g.r) * 4;
    const T* row = Bl + (size_t)i * g.d;
    float a[4] = {0.f, 0.f, 0.f, 0.f};
    if ((g.d & 7) == 0) {
      for (int e = 0; e < g.d; e += 8) {
        float v[8];
        Vec8<T>::load(row + e, v);
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          if (j0 + jj < g.g) {
            const float* qq = qs + (j0 + jj) * g.d + e;
#pragma unroll
            for (int x = 0; x < 8; ++x) a[jj] = fmaf(v[x], qq[x], a[jj]);
          }
        }
      }
    } else {
      for (int e = 0; e < g.d; ++e) {
        const float v = to_f(row[e]);
#pragma unroll
        for (int jj = 0; jj < 4; ++jj)
          if (j0 + jj < g.g) a[jj] = fmaf(v, qs[(j0 + jj) * g.d + e], a[jj]);
      }
    }
#pragma unroll
    for (int jj = 0; jj < 4; ++jj)
      if (j0 + jj < g.g) qt[(j0 + jj) * g.r + i] = a[jj];
  }
  __syncthreads();
  for (int i = tid; i < g.r; i += blockDim.x) {
    float s = 0.f;
    for (int j = 0; j < g.g; ++j) s += qt[j * g.r + i];
    qsum[i] = s;
  }
  for (int i = tid; i < g.g * g.r; i += blockDim.x)
    sc.qt[(size_t)u * g.g * g.r + i] = qt[i] * g.qk_scale_log2;
  if (tc_q_mode) {
    // 16 rows (query heads padded with zeros) of r 16-bit values for the MMA B operand
    for (int i = tid; i < 16 * g.r; i += blockDim.x) {
      int j = i / g.r;
      float v = j < g.g ? qt[i] * g.qk_scale_log2 : 0.f;
      if (tc_q_mode == 1)
        reinterpret_cast<__nv_bfloat16*>(sc.qt_tc)[(size_t)u * 16 * g.r + i] = __float2bfloat16_rn(v);
      else
        reinterpret_cast<__half*>(sc.qt_tc)[(size_t)u * 16 * g.r + i] = __float2half_rn(v);
    }
  }
  __syncthreads();

  // --- chunk scores over live chunks: one thread per chunk
  const int16_t* slot = cb.slot ? cb.slot + (((size_t)un.b * NG + grp) * g.Hkv + un.hkv) * g.nC : nullptr;
  const T* summ = reinterpret_cast<const T*>(cb.summary) +
                  (((size_t)un.b * NG + grp) * g.Hkv + un.hkv) * (size_t)g.nL * g.r;
  const float inv_sqrt_d = rsqrtf((float)g.d);
  for (int c = tid; c < g.nC; c += blockDim.x) {
    const int sl = slot ? (int)slot[c] : c;
    float s = -INFINITY;
    if (sl >= 0 && sl < g.nL) {
      s = row_dot(summ + (size_t)sl * g.r, qsum, g.r) * inv_sqrt_d;
    } else if (sl >= g.nL) {
      atomicOr(sc.err, ERR_SLOT);
    }
    sc_s[c] = s;
    keys[c] = ((unsigned long long)(~float_order(s)) << 32) | (unsigned)c;
  }
  for (int c = g.nC + tid; c < nCp; c += blockDim.x) keys[c] = ~0ull;
  __syncthreads();
  if (scores_out) {
    float* so = scores_out + ((size_t)(un.li * g.B + un.b) * g.Hkv + un.hkv) * g.nC;
    for (int c = tid; c < g.nC; c += blockDim.x) so[c] = sc_s[c];
  }

  // --- top-k: order by (descending score, ascending id); keep k; ids ascending
  int32_t* sel_slot = sc.sel_slot + (size_t)u * g.k;
  int32_t* sel_id = sc.sel_id + (size_t)u * g.k;
  int32_t* sel_user = sel_out ? sel_out + ((size_t)(un.li * g.B + un.b) * g.Hkv + un.hkv) * g.k : nullptr;
  if (rank_topk) {
    // rank of each key among all keys (keys are distinct: the id is in the low bits)
    for (int c = tid; c < g.nC; c += blockDim.x) {
      const unsigned long long kc = keys[c];
      int rank = 0;
#pragma unroll 8
      for (int c2 = 0; c2 < g.nC; ++c2) rank += keys[c2] < kc ? 1 : 0;
      selv[c] = rank < g.k ? 1 : 0;
    }
    __syncthreads();
    // position among the selected ids = number of selected ids below it
    for (int c = tid; c < g.nC; c += blockDim.x) {
      if (!selv[c]) continue;
      int pos = 0;
      for (int c2 = 0; c2 < c; ++c2) pos += selv[c2];
      int sl = slot ? (int)slot[c] : c;
      if (sl < 0 || sl >= g.nL) {
        atomicOr(sc.err, ERR_SELECT);
        sl = 0;
      }
      sel_slot[pos] = sl;
      sel_id[pos] = c;
      if (sel_user) sel_user[pos] = c;
    }
  } else {
    bitonic_sort(keys, nCp);
    for (int i = tid; i < kp; i += blockDim.x) selv[i] = i < g.k ? (int)(keys[i] & 0xffffffffu) : 0x7fffffff;
    __syncthreads();
    for (int i = tid; i < kp; i += blockDim.x) keys[i] = (unsigned long long)(unsigned)selv[i];
    __syncthreads();
    bitonic_sort(keys, kp);
    for (int i = tid; i < g.k; i += blockDim.x) {
      const int id = (int)keys[i];
      int sl = slot ? (int)slot[id] : id;
      if (sl < 0 || sl >= g.nL) {
        atomicOr(sc.err, ERR_SELECT);
        sl = 0;
      }
      sel_slot[i] = sl;
      sel_id[i] = id;
      if (sel_user) sel_user[i] = id;
    }
  }
  if (!do_tail) return;

  // --- raw tail: partial softmax over its tokens (online, blocks of kTailBlock tokens)
  int tl = cb.tail_len[un.b];
  if (tl < 0 || tl > g.T) {
    if (tid == 0) atomicOr(sc.err, ERR_TAIL_LEN);
    tl = tl < 0 ? 0 : g.T;
  }
  for (int i = tid; i < g.g * g.d; i += blockDim.x) acc[i] = 0.f;
  if (tid < g.g) {
    mrun[tid] = -INFINITY;
    lrun[tid] = 0.f;
  }
  __syncthreads();
  const size_t toff = (((size_t)un.b * g.L + l) * g.Hkv + un.hkv) * (size_t)g.T * g.d;
  const T* tk = reinterpret_cast<const T*>(cb.tail_k) + toff;
  const T* tv = reinterpret_cast<const T*>(cb.tail_v) + toff;
  for (int t0 = 0; t0 < tl; t0 += kTailBlock) {
    const int nb = min(kTailBlock, tl - t0);
    // logits: one thread per token, all query heads of the unit
    for (int t = tid; t < nb; t += blockDim.x) {
      const T* row = tk + (size_t)(t0 + t) * g.d;
      for (int j = 0; j < g.g; ++j) lg[j * kTailBlock + t] = row_dot(row, qs + j * g.d, g.d) * g.qk_scale_log2;
    }
    __syncthreads();
    for (int j = warp; j < g.g; j += nwarp) {
      float m = -INFINITY;
      for (int t = lane; t < nb; t += 32) m = fmaxf(m, lg[j * kTailBlock + t]);
      m = warp_max(m);
      const float mnew = fmaxf(mrun[j], m);
      float s = 0.f;
      for (int t = lane; t < nb; t += 32) {
        const float p = exp2f(lg[j * kTailBlock + t] - mnew);
        lg[j * kTailBlock + t] = p;
        s += p;
      }
      s = warp_sum(s);
      if (lane == 0) {
        const float a = exp2f(mrun[j] - mnew);  // 0 when mrun = -inf
        alpha[j] = a;
        lrun[j] = lrun[j] * a + s;
        mrun[j] = mnew;
      }
    }
    __syncthreads();
    for (int i = tid; i < g.g * g.d; i += blockDim.x) {
      const int j = i / g.d, dd = i % g.d;
      const float* p = lg + j * kTailBlock;
      const T* col = tv + (size_t)t0 * g.d + dd;
      float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
      int t = 0;
      for (; t + 4 <= nb; t += 4) {
        a0 = fmaf(p[t], to_f(col[(size_t)t * g.d]), a0);
        a1 = fmaf(p[t + 1], to_f(col[(size_t)(t + 1) * g.d]), a1);
        a2 = fmaf(p[t + 2], to_f(col[(size_t)(t + 2) * g.d]), a2);
        a3 = fmaf(p[t + 3], to_f(col[(size_t)(t + 3) * g.d]), a3);
      }
      for (; t < nb; ++t) a0 = fmaf(p[t], to_f(col[(size_t)t * g.d]), a0);
      acc[i] = acc[i] * alpha[j] + ((a0 + a1) + (a2 + a3));
    }
    __syncthreads();
  }
  float* rec = sc.tail_part + (size_t)u * g.tail_stride;
  for (int i = tid; i < g.g; i += blockDim.x) {
    rec[i] = mrun[i];
    rec[g.g + i] = lrun[i];
  }
  for (int i = tid; i < g.g * g.d; i += blockDim.x) rec[2 * g.g + i] = acc[i];
}

size_t select_smem_bytes(const Geom& g) {
  const int nCp = g.nC <= kRankMax ? g.nC : next_pow2(g.nC);
  int kp = 1;
  while (kp < g.k) kp <<= 1;
  const size_t floats = (size_t)g.g * g.d + (size_t)g.g * g.r + g.r + g.nC +
                        (size_t)(kp > g.nC ? kp : g.nC) + (size_t)g.g * kTailBlock +
                        (size_t)g.g * g.d + 3 * g.g;
  return (size_t)nCp * 8 + floats * 4;
}

}  // namespace

cudaError_t launch_select(const Geom& g, const CacheBuffers& cb, const Scratch& sc, int dtype,
                          const void* q, float* scores_out, int32_t* sel_out, int tc_q_mode,
                          bool tail, cudaStream_t s) {
  const size_t smem = select_smem_bytes(g);
  if (smem > 227 * 1024) return cudaErrorInvalidConfiguration;
  if (dtype == LOWRAM_F32) {
    auto k = select_kernel<float>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<g.U, kThreads, smem, s>>>(g, cb, sc, static_cast<const float*>(q), scores_out, sel_out,
                                  tc_q_mode, tail ? 1 : 0);
  } else {
    auto k = select_kernel<__nv_bfloat16>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<g.U, kThreads, smem, s>>>(g, cb, sc, static_cast<const __nv_bfloat16*>(q), scores_out,
                                  sel_out, tc_q_mode, tail ? 1 : 0);
  }
  return cudaGetLastError();
}

}  // namespace lowram
