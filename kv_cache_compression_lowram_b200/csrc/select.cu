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
#include "lowram_internal.cuh"

namespace lowram {
namespace {

constexpr int kThreads = 256;
constexpr int kTailBlock = 128;

__device__ __forceinline__ uint32_t float_order(float x) {
  uint32_t u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ int next_pow2(int n) {
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
  const int nCp = next_pow2(g.nC);
  const int kp = next_pow2(g.k);

  unsigned long long* keys = reinterpret_cast<unsigned long long*>(smem_raw);  // [nCp]
  float* qs = reinterpret_cast<float*>(keys + nCp);                             // [g][d]
  float* qt = qs + g.g * g.d;                                                   // [g][r]
  float* qsum = qt + g.g * g.r;                                                 // [r]
  float* sc_s = qsum + g.r;                                                     // [nC]
  int* selv = reinterpret_cast<int*>(sc_s + g.nC);                              // [kp]
  float* lg = reinterpret_cast<float*>(selv + kp);                              // [g][128]
  float* acc = lg + g.g * kTailBlock;                                           // [g][d]
  float* mrun = acc + g.g * g.d;                                                // [g]
  float* lrun = mrun + g.g;                                                     // [g]
  float* alpha = lrun + g.g;                                                    // [g]

  // --- the unit's queries
  const size_t qoff = ((size_t)(un.li * g.B + un.b) * g.Hq + (size_t)un.hkv * g.g) * g.d;
  for (int i = tid; i < g.g * g.d; i += blockDim.x) qs[i] = to_f(q[qoff + i]);
  __syncthreads();

  // --- qt_j = B_l q_j (coefficient space), one warp per basis row
  const T* Bl = reinterpret_cast<const T*>(cb.basis) + ((size_t)l * g.Hkv + un.hkv) * g.r * g.d;
  for (int i = warp; i < g.r; i += nwarp) {
    const T* row = Bl + (size_t)i * g.d;
    for (int j = 0; j < g.g; ++j) {
      float a = 0.f;
      for (int dd = lane; dd < g.d; dd += 32) a = fmaf(to_f(row[dd]), qs[j * g.d + dd], a);
      a = warp_sum(a);
      if (lane == 0) qt[j * g.r + i] = a;
    }
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

  // --- chunk scores over live chunks
  const int16_t* slot = cb.slot ? cb.slot + (((size_t)un.b * NG + grp) * g.Hkv + un.hkv) * g.nC : nullptr;
  const T* summ = reinterpret_cast<const T*>(cb.summary) +
                  (((size_t)un.b * NG + grp) * g.Hkv + un.hkv) * (size_t)g.nL * g.r;
  const float inv_sqrt_d = rsqrtf((float)g.d);
  for (int c = warp; c < g.nC; c += nwarp) {
    int sl = slot ? (int)slot[c] : c;
    float s = -INFINITY;
    if (sl >= 0 && sl < g.nL) {
      const T* row = summ + (size_t)sl * g.r;
      float a = 0.f;
      for (int i = lane; i < g.r; i += 32) a = fmaf(qsum[i], to_f(row[i]), a);
      a = warp_sum(a);
      s = a * inv_sqrt_d;
    } else if (sl >= g.nL && lane == 0) {
      atomicOr(sc.err, ERR_SLOT);
    }
    if (lane == 0) sc_s[c] = s;
  }
  __syncthreads();
  if (scores_out) {
    float* so = scores_out + ((size_t)(un.li * g.B + un.b) * g.Hkv + un.hkv) * g.nC;
    for (int c = tid; c < g.nC; c += blockDim.x) so[c] = sc_s[c];
  }

  // --- top-k: sort (descending score, ascending id), keep k, sort the ids ascending
  for (int c = tid; c < nCp; c += blockDim.x) {
    keys[c] = c < g.nC ? ((unsigned long long)(~float_order(sc_s[c])) << 32) | (unsigned)c
                       : ~0ull;
  }
  __syncthreads();
  bitonic_sort(keys, nCp);
  for (int i = tid; i < kp; i += blockDim.x) selv[i] = i < g.k ? (int)(keys[i] & 0xffffffffu) : 0x7fffffff;
  __syncthreads();
  // ascending ids (kp <= nCp, reuse the key buffer)
  for (int i = tid; i < kp; i += blockDim.x) keys[i] = (unsigned long long)(unsigned)selv[i];
  __syncthreads();
  bitonic_sort(keys, kp);
  for (int i = tid; i < g.k; i += blockDim.x) {
    int id = (int)keys[i];
    int sl = slot ? (int)slot[id] : id;
    if (sl < 0 || sl >= g.nL) {
      atomicOr(sc.err, ERR_SELECT);
      sl = 0;
    }
    sc.sel_slot[(size_t)u * g.k + i] = sl;
    sc.sel_id[(size_t)u * g.k + i] = id;
    if (sel_out) sel_out[((size_t)(un.li * g.B + un.b) * g.Hkv + un.hkv) * g.k + i] = id;
  }
  if (!do_tail) return;

  // --- raw tail: partial softmax over its tokens (online, blocks of 128 tokens)
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
    for (int t = warp; t < nb; t += nwarp) {
      const T* row = tk + (size_t)(t0 + t) * g.d;
      for (int j = 0; j < g.g; ++j) {
        float a = 0.f;
        for (int dd = lane; dd < g.d; dd += 32) a = fmaf(to_f(row[dd]), qs[j * g.d + dd], a);
        a = warp_sum(a);
        if (lane == 0) lg[j * kTailBlock + t] = a * g.qk_scale_log2;
      }
    }
    __syncthreads();
    for (int j = warp; j < g.g; j += nwarp) {
      float m = -INFINITY;
      for (int t = lane; t < nb; t += 32) m = fmaxf(m, lg[j * kTailBlock + t]);
      m = warp_max(m);
      const float mnew = fmaxf(mrun[j], m);
      float s = 0.f;
      for (int t = lane; t < nb; t += 32) {
        float p = exp2f(lg[j * kTailBlock + t] - mnew);
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
      float a = acc[i] * alpha[j];
      for (int t = 0; t < nb; ++t) a = fmaf(lg[j * kTailBlock + t], to_f(tv[(size_t)(t0 + t) * g.d + dd]), a);
      acc[i] = a;
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
  int nCp = 1;
  while (nCp < g.nC) nCp <<= 1;
  int kp = 1;
  while (kp < g.k) kp <<= 1;
  size_t floats = (size_t)g.g * g.d + (size_t)g.g * g.r + g.r + g.nC + kp +
                  (size_t)g.g * kTailBlock + (size_t)g.g * g.d + 3 * g.g;
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
