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
              int do_tail, SelCand cand) {
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
  const int16_t* slot = cb.slot ? cb.slot + (((size_t)un.b * NG + grp) * g.Hkv + un.hkv) * g.nCs : nullptr;
  const T* summ = reinterpret_cast<const T*>(cb.summary) +
                  (((size_t)un.b * NG + grp) * g.Hkv + un.hkv) * (size_t)g.nLs * g.r;
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
  const size_t ui = ((size_t)(un.li * g.B + un.b) * g.Hkv + un.hkv);   // the caller's unit index
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
      if (cand.score) {
        cand.score[ui * g.k + pos] = sc_s[c];
        cand.id[ui * g.k + pos] = c + cand.offset;
      }
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
      if (cand.score) {
        cand.score[ui * g.k + i] = sc_s[id];
        cand.id[ui * g.k + i] = id + cand.offset;
      }
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

// ---------------------------------------------------------------------------- fast path
// The same computation for the common shapes (bf16, d = 128, r in {64, 128}, g in {4, 8},
// at most 1024 chunks), one CTA of 8 warps per unit.  The chunk selection and the raw tail's
// partial softmax do not depend on each other: warps 0-3 project the queries, score the
// chunks and select, warps 4-7 run the tail, each group with its own named barrier.  The
// top-k needs no barrier at all: one warp holds every chunk's order key (nC / 32 per lane)
// and finds the k-th largest by a bitwise binary search with warp-wide counts, then takes
// the keys equal to it in ascending chunk id.  The tail's value rows are staged into shared
// memory by cp.async at entry, so their latency hides under the logits.  Shared memory and
// registers stay small (several units per SM), so a whole call runs in about one wave.
constexpr int kSelThreads = 256;     // warps 0-3: selection; warps 4-7: raw tail
constexpr int kSelTB = 128;          // tail tokens per block (one per tail thread)

// 16-byte asynchronous copy global -> shared (zero-filled when !valid); completes at the
// next cp.async.wait_group.
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc, bool valid) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(gsrc), "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void bar_named(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }

// Exclusive prefix sum over the lanes of a warp.
__device__ __forceinline__ int warp_excl_scan(int v) {
  const int lane = threadIdx.x & 31;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  return x - v;
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4& w, float (&v)[8]) {
  const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(ww[i] << 16);
    v[2 * i + 1] = __uint_as_float(ww[i] & 0xffff0000u);
  }
}

template <int R, int GQ, int NPL>
struct SelSmem {
  float qs[GQ][128];              // the unit's queries
  float qsum[R];                  // sum_j B_l q_j
  float score[NPL * 32];          // chunk scores (ids >= nC unused)
  float p[kSelTB][GQ];            // tail probabilities of the current block, token-major
  float red_max[4][GQ];           // per tail warp: block maxima, then block sums
  float red_sum[4][GQ];
  float pv[GQ][128];              // the second token half's P.V sums
  __align__(16) __nv_bfloat16 v[kSelTB][128];   // the block's tail values
};

template <int R, int GQ, int NPL>
__global__ void __launch_bounds__(kSelThreads, GQ <= 4 ? 3 : 2)
select_warp_kernel(Geom g, CacheBuffers cb, Scratch sc, const __nv_bfloat16* __restrict__ q,
                   float* __restrict__ scores_out, int32_t* __restrict__ sel_out, int tc_q_mode,
                   int do_tail, SelCand cand) {
  constexpr int D = 128;
  using SM = SelSmem<R, GQ, NPL>;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SM& sm = *reinterpret_cast<SM*>(smem_raw);
  const int u = blockIdx.x;
  const Unit un = unit_of(g, u);
  const int l = g.layer0 + un.li;
  const int grp = l / g.G;
  const int NG = g.L / g.G;
  const int nC = g.nC;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // tail set-up first: its value rows start streaming into shared memory right away
  int tl = 0;
  const size_t toff = (((size_t)un.b * g.L + l) * g.Hkv + un.hkv) * (size_t)g.T * D;
  const __nv_bfloat16* tk = reinterpret_cast<const __nv_bfloat16*>(cb.tail_k) + toff;
  const __nv_bfloat16* tv = reinterpret_cast<const __nv_bfloat16*>(cb.tail_v) + toff;
  const int tt = tid - 128;   // tail thread index (warps 4-7)
  auto stage_v = [&](int t0) {   // rows t0 .. t0+127 (zero past the tail)
#pragma unroll 4
    for (int k = 0; k < 16; ++k) {
      const int it = tt + k * 128, t = it >> 4, e = it & 15;
      const bool in = t0 + t < tl;
      cp_async16(&sm.v[t][e * 8], in ? tv + (size_t)(t0 + t) * D + e * 8 : tv, in);
    }
    cp_async_commit();
  };
  if (warp >= 4 && do_tail) {
    tl = cb.tail_len[un.b];
    if (tl < 0 || tl > g.T) {
      if (tt == 0) atomicOr(sc.err, ERR_TAIL_LEN);
      tl = tl < 0 ? 0 : g.T;
    }
    if (tl > 0) stage_v(0);
  }

  // the unit's queries (GQ x 128 bf16, 16 bytes per thread)
  const size_t qoff = ((size_t)(un.li * g.B + un.b) * g.Hq + (size_t)un.hkv * GQ) * D;
  if (tid < GQ * D / 8) {
    float v[8];
    bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(q + qoff) + tid), v);
#pragma unroll
    for (int i = 0; i < 8; ++i) (&sm.qs[0][0])[tid * 8 + i] = v[i];
  }
  __syncthreads();

  if (warp < 4) {
    // ============================================================ chunk selection
    const int st = tid;   // 0..127
    // --- qt_j = B_l q_j: PARTS threads per basis row
    {
      constexpr int PARTS = 128 / R;
      constexpr int SEG = D / PARTS;
      const int i = st / PARTS, part = st % PARTS;
      const uint4* row = reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(cb.basis) +
                                                        (((size_t)l * g.Hkv + un.hkv) * R + i) * D + part * SEG);
      float a[GQ];
#pragma unroll
      for (int j = 0; j < GQ; ++j) a[j] = 0.f;
#pragma unroll
      for (int h8 = 0; h8 < SEG / 32; ++h8) {   // 32 elements (4 loads) at a time
        uint4 w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) w[e] = __ldg(row + h8 * 4 + e);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float v[8];
          bf16x8_to_f32(w[e], v);
          const int col = part * SEG + (h8 * 4 + e) * 8;
#pragma unroll
          for (int j = 0; j < GQ; ++j) {
            const float4 q0 = *reinterpret_cast<const float4*>(&sm.qs[j][col]);
            const float4 q1 = *reinterpret_cast<const float4*>(&sm.qs[j][col + 4]);
            a[j] = fmaf(v[0], q0.x, fmaf(v[1], q0.y, fmaf(v[2], q0.z, fmaf(v[3], q0.w, a[j]))));
            a[j] = fmaf(v[4], q1.x, fmaf(v[5], q1.y, fmaf(v[6], q1.z, fmaf(v[7], q1.w, a[j]))));
          }
        }
      }
      if (PARTS == 2) {
#pragma unroll
        for (int j = 0; j < GQ; ++j) a[j] += __shfl_xor_sync(0xffffffffu, a[j], 1);
      }
      if (part == 0) {
        float s = 0.f;
#pragma unroll
        for (int j = 0; j < GQ; ++j) s += a[j];
        sm.qsum[i] = s;
#pragma unroll
        for (int j = 0; j < GQ; ++j) {
          const float v = a[j] * g.qk_scale_log2;
          sc.qt[((size_t)u * GQ + j) * R + i] = v;
          // rows >= GQ of the 16-row copy stay zero (cleared when the scratch is created)
          if (tc_q_mode == 1)
            reinterpret_cast<__nv_bfloat16*>(sc.qt_tc)[((size_t)u * 16 + j) * R + i] = __float2bfloat16_rn(v);
          else if (tc_q_mode == 2)
            reinterpret_cast<__half*>(sc.qt_tc)[((size_t)u * 16 + j) * R + i] = __float2half_rn(v);
        }
      }
    }
    bar_named(1, 128);

    // --- chunk scores: chunk ids st, st + 128, ...; the whole summary row loaded at once
    const int16_t* slot = cb.slot ? cb.slot + (((size_t)un.b * NG + grp) * g.Hkv + un.hkv) * g.nCs : nullptr;
    const __nv_bfloat16* summ = reinterpret_cast<const __nv_bfloat16*>(cb.summary) +
                                (((size_t)un.b * NG + grp) * g.Hkv + un.hkv) * (size_t)g.nLs * R;
    const float inv_sqrt_d = rsqrtf((float)D);
    float* so = scores_out ? scores_out + ((size_t)(un.li * g.B + un.b) * g.Hkv + un.hkv) * nC : nullptr;
#pragma unroll 1
    for (int c = st; c < NPL * 32; c += 128) {
      float s = -INFINITY;
      if (c < nC) {
        const int sl = slot ? (int)slot[c] : c;
        if (sl >= 0 && sl < g.nL) {
          const uint4* row = reinterpret_cast<const uint4*>(summ + (size_t)sl * R);
          float a0 = 0.f, a1 = 0.f;
#pragma unroll
          for (int h8 = 0; h8 < R / 64; ++h8) {   // 64 ranks (8 loads) at a time
            uint4 w[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) w[e] = __ldg(row + h8 * 8 + e);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              float v[8];
              bf16x8_to_f32(w[e], v);
              const int col = (h8 * 8 + e) * 8;
              const float4 q0 = *reinterpret_cast<const float4*>(&sm.qsum[col]);
              const float4 q1 = *reinterpret_cast<const float4*>(&sm.qsum[col + 4]);
              a0 = fmaf(v[0], q0.x, fmaf(v[2], q0.z, fmaf(v[4], q1.x, fmaf(v[6], q1.z, a0))));
              a1 = fmaf(v[1], q0.y, fmaf(v[3], q0.w, fmaf(v[5], q1.y, fmaf(v[7], q1.w, a1))));
            }
          }
          s = (a0 + a1) * inv_sqrt_d;
        } else if (sl >= g.nL) {
          atomicOr(sc.err, ERR_SLOT);
        }
        if (so) so[c] = s;
      }
      sm.score[c] = s;
    }
    bar_named(1, 128);
    if (warp != 0) return;

    // --- top-k (one warp): lane holds chunks lane*NPL .. lane*NPL + NPL-1; the order key
    // of a score is monotone in the score, and ids >= nC get key 0 (below every chunk's)
    uint32_t key[NPL];
#pragma unroll
    for (int i = 0; i < NPL; i += 4) {
      const float4 f = *reinterpret_cast<const float4*>(&sm.score[lane * NPL + i]);
      const float fv[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
      for (int x = 0; x < 4; ++x) key[i + x] = lane * NPL + i + x < nC ? float_order(fv[x]) : 0u;
    }
    // the k-th largest key: the largest T with #{key >= T} >= k, bit by bit from the top
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
    const int need_eq = g.k - (int)__reduce_add_sync(0xffffffffu, gt);   // >= 1 keys equal to T, lowest ids
    int eq_rank = warp_excl_scan(eq);
    uint32_t take = 0;
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
      if (key[i] > T) {
        take |= 1u << i;
      } else if (key[i] == T) {
        if (eq_rank < need_eq) take |= 1u << i;
        ++eq_rank;
      }
    }
    int pos = warp_excl_scan(__popc(take));
    int32_t* sel_slot = sc.sel_slot + (size_t)u * g.k;
    int32_t* sel_id = sc.sel_id + (size_t)u * g.k;
    int32_t* sel_user = sel_out ? sel_out + ((size_t)(un.li * g.B + un.b) * g.Hkv + un.hkv) * g.k : nullptr;
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
      if (take & (1u << i)) {
        const int c = lane * NPL + i;
        int sl = slot ? (int)slot[c] : c;
        if (sl < 0 || sl >= g.nL) {
          atomicOr(sc.err, ERR_SELECT);
          sl = 0;
        }
        if (pos < g.k) {
          sel_slot[pos] = sl;
          sel_id[pos] = c;
          if (sel_user) sel_user[pos] = c;
          if (cand.score) {
            const size_t ui = ((size_t)(un.li * g.B + un.b) * g.Hkv + un.hkv) * g.k + pos;
            cand.score[ui] = sm.score[c];
            cand.id[ui] = c + cand.offset;
          }
        }
        ++pos;
      }
    }
    return;
  }
  if (!do_tail) return;

  // ============================================================ raw tail
  // Blocks of 128 tokens: thread tt's logits are token t0 + tt's (all heads); its P.V share
  // is dimension pair dp over one half th of the block's tokens.
  const int tw = warp - 4;
  const int dp = tt & 63, th = tt >> 6;
  float m_run[GQ], l_run[GQ], acc[GQ][2];
#pragma unroll
  for (int j = 0; j < GQ; ++j) {
    m_run[j] = -INFINITY;
    l_run[j] = 0.f;
    acc[j][0] = acc[j][1] = 0.f;
  }
#pragma unroll 1
  for (int t0 = 0; t0 < tl; t0 += kSelTB) {
    const int nb = min(kSelTB, tl - t0);
    float lg[GQ];
#pragma unroll
    for (int j = 0; j < GQ; ++j) lg[j] = -INFINITY;
    if (tt < nb) {
      const uint4* krow = reinterpret_cast<const uint4*>(tk + (size_t)(t0 + tt) * D);
      float a[GQ];
#pragma unroll
      for (int j = 0; j < GQ; ++j) a[j] = 0.f;
#pragma unroll
      for (int h8 = 0; h8 < 4; ++h8) {   // 32 dims (4 loads) at a time: the running state stays in registers
        uint4 w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) w[e] = __ldg(krow + h8 * 4 + e);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float v[8];
          bf16x8_to_f32(w[e], v);
          const int col = (h8 * 4 + e) * 8;
#pragma unroll
          for (int j = 0; j < GQ; ++j) {
            const float4 q0 = *reinterpret_cast<const float4*>(&sm.qs[j][col]);
            const float4 q1 = *reinterpret_cast<const float4*>(&sm.qs[j][col + 4]);
            a[j] = fmaf(v[0], q0.x, fmaf(v[1], q0.y, fmaf(v[2], q0.z, fmaf(v[3], q0.w, a[j]))));
            a[j] = fmaf(v[4], q1.x, fmaf(v[5], q1.y, fmaf(v[6], q1.z, fmaf(v[7], q1.w, a[j]))));
          }
        }
      }
#pragma unroll
      for (int j = 0; j < GQ; ++j) lg[j] = a[j] * g.qk_scale_log2;
    }
#pragma unroll
    for (int j = 0; j < GQ; ++j) {
      const float mx = warp_max(lg[j]);
      if (lane == 0) sm.red_max[tw][j] = mx;
    }
    bar_named(2, 128);
    float alpha[GQ];
#pragma unroll
    for (int j = 0; j < GQ; ++j) {
      const float mb = fmaxf(fmaxf(sm.red_max[0][j], sm.red_max[1][j]), fmaxf(sm.red_max[2][j], sm.red_max[3][j]));
      const float mn = fmaxf(m_run[j], mb);   // finite: the block has at least one token
      alpha[j] = exp2f(m_run[j] - mn);        // 0 while m_run = -inf
      const float p = exp2f(lg[j] - mn);      // 0 past the tail
      sm.p[tt][j] = p;
      const float ps = warp_sum(p);
      if (lane == 0) sm.red_sum[tw][j] = ps;
      m_run[j] = mn;
    }
    cp_async_wait_all();   // this thread's copies of the block's value rows (the barrier shares them)
    bar_named(2, 128);
#pragma unroll
    for (int j = 0; j < GQ; ++j) {
      l_run[j] = l_run[j] * alpha[j] + (sm.red_sum[0][j] + sm.red_sum[1][j]) + (sm.red_sum[2][j] + sm.red_sum[3][j]);
      acc[j][0] *= alpha[j];
      acc[j][1] *= alpha[j];
    }
    const int tb = th * (kSelTB / 2), te = min(tb + kSelTB / 2, nb);
#pragma unroll 4
    for (int t = tb; t < te; ++t) {
      const uint32_t w = *reinterpret_cast<const uint32_t*>(&sm.v[t][2 * dp]);
      const float v0 = __uint_as_float(w << 16), v1 = __uint_as_float(w & 0xffff0000u);
#pragma unroll
      for (int j = 0; j < GQ; j += 4) {
        const float4 pj = *reinterpret_cast<const float4*>(&sm.p[t][j]);
        acc[j][0] = fmaf(pj.x, v0, acc[j][0]);
        acc[j][1] = fmaf(pj.x, v1, acc[j][1]);
        acc[j + 1][0] = fmaf(pj.y, v0, acc[j + 1][0]);
        acc[j + 1][1] = fmaf(pj.y, v1, acc[j + 1][1]);
        acc[j + 2][0] = fmaf(pj.z, v0, acc[j + 2][0]);
        acc[j + 2][1] = fmaf(pj.z, v1, acc[j + 2][1]);
        acc[j + 3][0] = fmaf(pj.w, v0, acc[j + 3][0]);
        acc[j + 3][1] = fmaf(pj.w, v1, acc[j + 3][1]);
      }
    }
    if (t0 + kSelTB < tl) {   // the next block's value rows, once every thread is done with these
      bar_named(2, 128);
      stage_v(t0 + kSelTB);
    }
  }
  // the two token halves' sums, then the tail record (log2-domain max, sum, sums per head)
  if (th == 1) {
#pragma unroll
    for (int j = 0; j < GQ; ++j) {
      sm.pv[j][2 * dp] = acc[j][0];
      sm.pv[j][2 * dp + 1] = acc[j][1];
    }
  }
  bar_named(2, 128);
  float* rec = sc.tail_part + (size_t)u * g.tail_stride;
  if (th == 0) {
#pragma unroll
    for (int j = 0; j < GQ; ++j) {
      rec[2 * GQ + j * D + 2 * dp] = acc[j][0] + sm.pv[j][2 * dp];
      rec[2 * GQ + j * D + 2 * dp + 1] = acc[j][1] + sm.pv[j][2 * dp + 1];
    }
  }
  if (tt < GQ) {
    rec[tt] = m_run[tt];
    rec[GQ + tt] = l_run[tt];
  }
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

namespace {

template <int R, int GQ, int NPL>
cudaError_t launch_select_warp(const Geom& g, const CacheBuffers& cb, const Scratch& sc, const void* q,
                               float* scores_out, int32_t* sel_out, int tc_q_mode, bool tail, cudaStream_t s,
                               SelCand cand) {
  using SM = SelSmem<R, GQ, NPL>;
  auto k = select_warp_kernel<R, GQ, NPL>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(SM));
  if (e != cudaSuccess) return e;
  k<<<g.U, kSelThreads, sizeof(SM), s>>>(g, cb, sc, static_cast<const __nv_bfloat16*>(q), scores_out, sel_out,
                                         tc_q_mode, tail ? 1 : 0, cand);
  return cudaGetLastError();
}

template <int R, int GQ>
cudaError_t launch_select_fast(const Geom& g, const CacheBuffers& cb, const Scratch& sc, const void* q,
                               float* scores_out, int32_t* sel_out, int tc_q_mode, bool tail, cudaStream_t s,
                               SelCand cand) {
  if (g.nC <= 256) return launch_select_warp<R, GQ, 8>(g, cb, sc, q, scores_out, sel_out, tc_q_mode, tail, s, cand);
  if (g.nC <= 512) return launch_select_warp<R, GQ, 16>(g, cb, sc, q, scores_out, sel_out, tc_q_mode, tail, s, cand);
  return launch_select_warp<R, GQ, 32>(g, cb, sc, q, scores_out, sel_out, tc_q_mode, tail, s, cand);
}

}  // namespace

cudaError_t launch_select(const Geom& g, const CacheBuffers& cb, const Scratch& sc, int dtype,
                          const void* q, float* scores_out, int32_t* sel_out, int tc_q_mode,
                          bool tail, cudaStream_t s, SelCand cand) {
  if (dtype == LOWRAM_BF16 && g.d == 128 && g.nC <= kRankMax && (reinterpret_cast<uintptr_t>(q) & 15) == 0) {
#define LOWRAM_SELECT_FAST(RR, GG) \
    if (g.r == RR && g.g == GG) return launch_select_fast<RR, GG>(g, cb, sc, q, scores_out, sel_out, tc_q_mode, tail, s, cand);
    LOWRAM_SELECT_FAST(128, 4)
    LOWRAM_SELECT_FAST(128, 8)
    LOWRAM_SELECT_FAST(64, 4)
    LOWRAM_SELECT_FAST(64, 8)
#undef LOWRAM_SELECT_FAST
  }
  const size_t smem = select_smem_bytes(g);
  if (smem > 227 * 1024) return cudaErrorInvalidConfiguration;
  if (dtype == LOWRAM_F32) {
    auto k = select_kernel<float>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<g.U, kThreads, smem, s>>>(g, cb, sc, static_cast<const float*>(q), scores_out, sel_out,
                                  tc_q_mode, tail ? 1 : 0, cand);
  } else {
    auto k = select_kernel<__nv_bfloat16>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<g.U, kThreads, smem, s>>>(g, cb, sc, static_cast<const __nv_bfloat16*>(q), scores_out,
                                  sel_out, tc_q_mode, tail ? 1 : 0, cand);
  }
  return cudaGetLastError();
}

}  // namespace lowram
