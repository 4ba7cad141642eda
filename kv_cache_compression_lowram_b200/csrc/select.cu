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

// ---------------------------------------------------------------------------- fast path
// The same computation for the common shapes (bf16, d = 128, r in {64, 128}, g in {4, 8},
// at most kRankMax chunks).  The chunk selection (projection, scores, top-k) and the raw
// tail's partial softmax do not depend on each other, so each runs in its own half of a
// 512-thread CTA with its own named barrier; only the queries are shared.  Every thread
// issues all of its global loads before it uses any of them, basis and summary rows are
// split across threads, the raw tail is staged in 64-token blocks through a two-buffer
// cp.async ring (rows padded by 16 bytes against bank conflicts), and the selected ids
// are placed with a ballot scan.
constexpr int kFastTB = 64;               // tail tokens per staged block
constexpr int kFastHalf = 256;            // threads per half of the fast kernel
constexpr int kFastThreads = 2 * kFastHalf;

// 16-byte asynchronous copy global -> shared (zero-filled when !valid); completes at the
// next cp.async.wait_group.
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc, bool valid) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(gsrc), "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_one() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }
// barrier among the 256 threads of one half (ids 1 and 2; 0 is __syncthreads)
__device__ __forceinline__ void half_sync(int id) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(kFastHalf) : "memory");
}
constexpr int kRowPad = 8;                // bf16 elements of padding per staged tail row

template <int R, int GQ>
struct FastSmem {
  static constexpr int D = 128;
  static constexpr int KROW = D + kRowPad;
  static constexpr size_t TBUF = (size_t)kFastTB * KROW * 2 + (size_t)kFastTB * D * 2;   // K + V block
  static constexpr size_t bytes(int nC) {
    return (size_t)nC * 8                      // keys
           + (size_t)GQ * D * 4                // qs
           + (size_t)GQ * R * 4                // qt
           + (size_t)R * 4                     // qsum
           + (size_t)nC * 4                    // scores
           + (size_t)nC * 4                    // selected flags
           + 256 * 4                           // radix histogram
           + 2 * TBUF                          // two tail blocks
           + (size_t)GQ * kFastTB * 4          // logits / probabilities
           + (size_t)4 * GQ * D * 4            // P.V partial sums of the 4 token quarters
           + (size_t)3 * GQ * 4 + 64;          // mrun, lrun, alpha, warp totals
  }
};

template <int R, int GQ>
__global__ void __launch_bounds__(kFastThreads)
select_fast_kernel(Geom g, CacheBuffers cb, Scratch sc, const __nv_bfloat16* __restrict__ q,
                   float* __restrict__ scores_out, int32_t* __restrict__ sel_out, int tc_q_mode,
                   int do_tail) {
  constexpr int D = 128;
  using SM = FastSmem<R, GQ>;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int u = blockIdx.x;
  const Unit un = unit_of(g, u);
  const int l = g.layer0 + un.li;
  const int grp = l / g.G;
  const int NG = g.L / g.G;
  const int nC = g.nC;
  const int tid = threadIdx.x;
  const bool tail_half = tid >= kFastHalf;
  const int ht = tid & (kFastHalf - 1), lane = ht & 31, warp = ht >> 5;   // within the half

  unsigned long long* keys = reinterpret_cast<unsigned long long*>(smem_raw);   // [nC]
  float* qs = reinterpret_cast<float*>(keys + nC);                               // [GQ][D]
  float* qt = qs + GQ * D;                                                       // [GQ][R]
  float* qsum = qt + GQ * R;                                                     // [R]
  float* sc_s = qsum + R;                                                        // [nC]
  int* selv = reinterpret_cast<int*>(sc_s + nC);                                 // [nC]
  int* hist = selv + nC;                                                         // [256]
  unsigned char* tbuf = reinterpret_cast<unsigned char*>(hist + 256);            // 2 x (K, V) blocks
  float* lg = reinterpret_cast<float*>(tbuf + 2 * SM::TBUF);                     // [GQ][TB]
  float* pv = lg + GQ * kFastTB;                                                 // [4][GQ][D]
  float* mrun = pv + 4 * GQ * D;                                                 // [GQ]
  float* lrun = mrun + GQ;
  float* alpha = lrun + GQ;
  int* wtot = reinterpret_cast<int*>(alpha + GQ);                                // [8]
  __shared__ int radix_state[2];

  int tl = do_tail ? cb.tail_len[un.b] : 0;
  if (tl < 0 || tl > g.T) {
    if (tid == 0) atomicOr(sc.err, ERR_TAIL_LEN);
    tl = tl < 0 ? 0 : g.T;
  }
  const size_t toff = (((size_t)un.b * g.L + l) * g.Hkv + un.hkv) * (size_t)g.T * D;
  const __nv_bfloat16* tk = reinterpret_cast<const __nv_bfloat16*>(cb.tail_k) + toff;
  const __nv_bfloat16* tv = reinterpret_cast<const __nv_bfloat16*>(cb.tail_v) + toff;
  // tail block b -> buffer b % 2: 16 x 16-byte pieces per row, 4 + 4 copies per thread of
  // the tail half; rows past the tail are zero-filled
  auto stage_block = [&](int blk) {
    __nv_bfloat16* kb = reinterpret_cast<__nv_bfloat16*>(tbuf + (blk & 1) * SM::TBUF);
    __nv_bfloat16* vb = kb + kFastTB * SM::KROW;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int it = ht + k * kFastHalf, t = it >> 4, e = it & 15;
      const int tt = blk * kFastTB + t;
      const bool in = tt < tl;
      cp_async16(kb + t * SM::KROW + e * 8, in ? tk + (size_t)tt * D + e * 8 : tk, in);
      cp_async16(vb + t * D + e * 8, in ? tv + (size_t)tt * D + e * 8 : tv, in);
    }
    cp_async_commit();
  };
  // the tail's first two blocks go to shared memory right away
  if (tail_half && do_tail) {
    stage_block(0);
    stage_block(1);
  }

  // --- the unit's queries (GQ x 128 bf16: one 16-byte load per thread for GQ <= 16)
  const size_t qoff = ((size_t)(un.li * g.B + un.b) * g.Hq + (size_t)un.hkv * GQ) * D;
  if (!tail_half && ht < GQ * D / 8) {
    float v[8];
    Vec8<__nv_bfloat16>::load(q + qoff + ht * 8, v);
#pragma unroll
    for (int i = 0; i < 8; ++i) qs[ht * 8 + i] = v[i];
  }
  __syncthreads();

  if (!tail_half) {
    // ============================================================ chunk selection
    // --- qt_j = B_l q_j: each basis row split over PARTS threads, all loads issued first
    {
      constexpr int PARTS = kFastHalf / R;         // 2 for r = 128, 4 for r = 64
      constexpr int SEG = D / PARTS;               // elements per thread
      const int i = ht / PARTS, part = ht % PARTS;
      const __nv_bfloat16* row = reinterpret_cast<const __nv_bfloat16*>(cb.basis) +
                                 (((size_t)l * g.Hkv + un.hkv) * R + i) * D + part * SEG;
      uint4 w[SEG / 8];
#pragma unroll
      for (int e = 0; e < SEG / 8; ++e) w[e] = __ldg(reinterpret_cast<const uint4*>(row) + e);
      float a[GQ];
#pragma unroll
      for (int j = 0; j < GQ; ++j) a[j] = 0.f;
#pragma unroll
      for (int e = 0; e < SEG / 8; ++e) {
        const uint32_t ww[4] = {w[e].x, w[e].y, w[e].z, w[e].w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const float v0 = __uint_as_float(ww[h] << 16), v1 = __uint_as_float(ww[h] & 0xffff0000u);
          const int col = part * SEG + e * 8 + 2 * h;
#pragma unroll
          for (int j = 0; j < GQ; ++j) a[j] = fmaf(v1, qs[j * D + col + 1], fmaf(v0, qs[j * D + col], a[j]));
        }
      }
#pragma unroll
      for (int j = 0; j < GQ; ++j) {
#pragma unroll
        for (int o = 1; o < PARTS; o <<= 1) a[j] += __shfl_xor_sync(0xffffffffu, a[j], o);
      }
      if (part == 0) {
#pragma unroll
        for (int j = 0; j < GQ; ++j) qt[j * R + i] = a[j];
      }
    }
    half_sync(1);
    for (int i = ht; i < R; i += kFastHalf) {
      float s = 0.f;
#pragma unroll
      for (int j = 0; j < GQ; ++j) s += qt[j * R + i];
      qsum[i] = s;
    }
    for (int i = ht; i < GQ * R; i += kFastHalf) sc.qt[(size_t)u * GQ * R + i] = qt[i] * g.qk_scale_log2;
    if (tc_q_mode) {
      for (int i = ht; i < 16 * R; i += kFastHalf) {
        const int j = i / R;
        const float v = j < GQ ? qt[i] * g.qk_scale_log2 : 0.f;
        if (tc_q_mode == 1)
          reinterpret_cast<__nv_bfloat16*>(sc.qt_tc)[(size_t)u * 16 * R + i] = __float2bfloat16_rn(v);
        else
          reinterpret_cast<__half*>(sc.qt_tc)[(size_t)u * 16 * R + i] = __float2half_rn(v);
      }
    }
    half_sync(1);

    // --- chunk scores: one thread per chunk, the whole summary row loaded at once
    const int16_t* slot = cb.slot ? cb.slot + (((size_t)un.b * NG + grp) * g.Hkv + un.hkv) * g.nCs : nullptr;
    const __nv_bfloat16* summ = reinterpret_cast<const __nv_bfloat16*>(cb.summary) +
                                (((size_t)un.b * NG + grp) * g.Hkv + un.hkv) * (size_t)g.nLs * R;
    const float inv_sqrt_d = rsqrtf((float)D);
    for (int c = ht; c < nC; c += kFastHalf) {
      const int sl = slot ? (int)slot[c] : c;
      float s = -INFINITY;
      if (sl >= 0 && sl < g.nL) {
        const uint4* row = reinterpret_cast<const uint4*>(summ + (size_t)sl * R);
        uint4 w[R / 8];
#pragma unroll
        for (int e = 0; e < R / 8; ++e) w[e] = __ldg(row + e);
        float a0 = 0.f, a1 = 0.f;
#pragma unroll
        for (int e = 0; e < R / 8; ++e) {
          const uint32_t ww[4] = {w[e].x, w[e].y, w[e].z, w[e].w};
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            a0 = fmaf(__uint_as_float(ww[h] << 16), qsum[e * 8 + 2 * h], a0);
            a1 = fmaf(__uint_as_float(ww[h] & 0xffff0000u), qsum[e * 8 + 2 * h + 1], a1);
          }
        }
        s = (a0 + a1) * inv_sqrt_d;
      } else if (sl >= g.nL) {
        atomicOr(sc.err, ERR_SLOT);
      }
      sc_s[c] = s;
      keys[c] = ((unsigned long long)(~float_order(s)) << 32) | (unsigned)c;
    }
    half_sync(1);
    if (scores_out) {
      float* so = scores_out + ((size_t)(un.li * g.B + un.b) * g.Hkv + un.hkv) * nC;
      for (int c = ht; c < nC; c += kFastHalf) so[c] = sc_s[c];
    }

    // --- top-k: radix select on the 32-bit order key (ascending = descending score), 8 bits
    // a pass, finds the k-th smallest key T and how many keys equal to T are still to take;
    // those go to the lowest ids.
    uint32_t prefix = 0;
    int kk = g.k;
#pragma unroll 1
    for (int shift = 24; shift >= 0; shift -= 8) {
      hist[ht] = 0;
      half_sync(1);
      for (int c = ht; c < nC; c += kFastHalf) {
        const uint32_t k32 = (uint32_t)(keys[c] >> 32);
        if (shift == 24 || (k32 >> (shift + 8)) == (prefix >> (shift + 8))) atomicAdd(&hist[(k32 >> shift) & 255], 1);
      }
      half_sync(1);
      const int hv = hist[ht];
      int v = hv;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int nv = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += nv;
      }
      if (lane == 31) wtot[warp] = v;
      half_sync(1);
      int woff = 0;
#pragma unroll
      for (int w2 = 0; w2 < kFastHalf / 32; ++w2) woff += w2 < warp ? wtot[w2] : 0;
      const int incl = v + woff, excl = incl - hv;
      if (excl < kk && incl >= kk) {
        radix_state[0] = ht;
        radix_state[1] = excl;
      }
      half_sync(1);
      prefix |= (uint32_t)radix_state[0] << shift;
      kk -= radix_state[1];
      half_sync(1);   // hist and wtot are rewritten by the next pass
    }
    // selected: key below T, or equal to T and among the kk lowest such ids
    {
      int eqrun = 0;
      for (int base = 0; base < nC; base += kFastHalf) {
        const int c = base + ht;
        const uint32_t k32 = c < nC ? (uint32_t)(keys[c] >> 32) : 0xffffffffu;
        const bool feq = c < nC && k32 == prefix;
        const unsigned beq = __ballot_sync(0xffffffffu, feq);
        if (lane == 0) wtot[warp] = __popc(beq);
        half_sync(1);
        int woff = 0, btot = 0;
#pragma unroll
        for (int w2 = 0; w2 < kFastHalf / 32; ++w2) {
          const int t2 = wtot[w2];
          woff += w2 < warp ? t2 : 0;
          btot += t2;
        }
        const int eqrank = eqrun + woff + __popc(beq & ((1u << lane) - 1u));
        if (c < nC) selv[c] = (k32 < prefix || (feq && eqrank < kk)) ? 1 : 0;
        eqrun += btot;
        half_sync(1);
      }
    }
    int32_t* sel_slot = sc.sel_slot + (size_t)u * g.k;
    int32_t* sel_id = sc.sel_id + (size_t)u * g.k;
    int32_t* sel_user = sel_out ? sel_out + ((size_t)(un.li * g.B + un.b) * g.Hkv + un.hkv) * g.k : nullptr;
    int run = 0;
    for (int base = 0; base < nC; base += kFastHalf) {
      const int c = base + ht;
      const int f = c < nC ? selv[c] : 0;
      const unsigned bal = __ballot_sync(0xffffffffu, f);
      if (lane == 0) wtot[warp] = __popc(bal);
      half_sync(1);
      int woff = 0, btot = 0;
#pragma unroll
      for (int w2 = 0; w2 < kFastHalf / 32; ++w2) {
        const int t2 = wtot[w2];
        woff += w2 < warp ? t2 : 0;
        btot += t2;
      }
      if (f) {
        const int pos = run + woff + __popc(bal & ((1u << lane) - 1u));
        int sl = slot ? (int)slot[c] : c;
        if (sl < 0 || sl >= g.nL) {
          atomicOr(sc.err, ERR_SELECT);
          sl = 0;
        }
        if (pos < g.k) {
          sel_slot[pos] = sl;
          sel_id[pos] = c;
          if (sel_user) sel_user[pos] = c;
        }
      }
      run += btot;
      half_sync(1);   // wtot is rewritten by the next round
    }
    return;
  }
  if (!do_tail) return;

  // ============================================================ raw tail
  // partial softmax over its tokens, block by block from the two-buffer ring
  constexpr int NACC = GQ * D / 2 / kFastHalf;   // (head, dim pair) sums per thread
  float accr[NACC][2];
#pragma unroll
  for (int n = 0; n < NACC; ++n) accr[n][0] = accr[n][1] = 0.f;
  if (ht < GQ) {
    mrun[ht] = -INFINITY;
    lrun[ht] = 0.f;
  }
  const int nblk = (tl + kFastTB - 1) / kFastTB;
  for (int bi = 0; bi < nblk; ++bi) {
    const int t0 = bi * kFastTB;
    const int nb = min(kFastTB, tl - t0);
    // block bi's copies (and, when it exists, block bi+1's may still be in flight)
    if (bi + 1 < nblk) cp_async_wait_one(); else cp_async_wait_all();
    half_sync(2);
    const __nv_bfloat16* kblk = reinterpret_cast<const __nv_bfloat16*>(tbuf + (bi & 1) * SM::TBUF);
    const __nv_bfloat16* vblk = kblk + kFastTB * SM::KROW;
    // logits: thread (token, GQ/4 heads)
    {
      constexpr int JPT = GQ / 4;
      const int t = ht & (kFastTB - 1), jb = ht / kFastTB;
      float a[JPT];
#pragma unroll
      for (int jj = 0; jj < JPT; ++jj) a[jj] = 0.f;
      const uint4* krow = reinterpret_cast<const uint4*>(kblk + t * SM::KROW);
#pragma unroll 4
      for (int e = 0; e < D / 8; ++e) {
        const uint4 w = krow[e];
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const float v0 = __uint_as_float(ww[h] << 16), v1 = __uint_as_float(ww[h] & 0xffff0000u);
#pragma unroll
          for (int jj = 0; jj < JPT; ++jj) {
            const float* qq = qs + (jb * JPT + jj) * D + e * 8 + 2 * h;
            a[jj] = fmaf(v1, qq[1], fmaf(v0, qq[0], a[jj]));
          }
        }
      }
#pragma unroll
      for (int jj = 0; jj < JPT; ++jj)
        lg[(jb * JPT + jj) * kFastTB + t] = t < nb ? a[jj] * g.qk_scale_log2 : -INFINITY;
    }
    half_sync(2);
    // online softmax update: one warp per head
    if (warp < GQ) {
      const int j = warp;
      const float x0 = lg[j * kFastTB + lane], x1 = lg[j * kFastTB + 32 + lane];
      const float mnew = fmaxf(mrun[j], warp_max(fmaxf(x0, x1)));
      const float p0 = exp2f(x0 - mnew), p1 = exp2f(x1 - mnew);
      lg[j * kFastTB + lane] = p0;
      lg[j * kFastTB + 32 + lane] = p1;
      const float ssum = warp_sum(p0 + p1);
      if (lane == 0) {
        const float a = exp2f(mrun[j] - mnew);   // 0 while mrun = -inf
        alpha[j] = a;
        lrun[j] = lrun[j] * a + ssum;
        mrun[j] = mnew;
      }
    }
    half_sync(2);
    // P.V over the block: thread (dim pair, quarter of the tokens), all heads
    {
      const int dp = ht & 63, tq = ht >> 6;
      float sacc[GQ][2];
#pragma unroll
      for (int j = 0; j < GQ; ++j) sacc[j][0] = sacc[j][1] = 0.f;
      const int tb = tq * (kFastTB / 4), te = min(tb + kFastTB / 4, nb);
      for (int t = tb; t < te; ++t) {
        const uint32_t w = reinterpret_cast<const uint32_t*>(vblk + t * D)[dp];
        const float v0 = __uint_as_float(w << 16), v1 = __uint_as_float(w & 0xffff0000u);
#pragma unroll
        for (int j = 0; j < GQ; ++j) {
          const float pj = lg[j * kFastTB + t];
          sacc[j][0] = fmaf(pj, v0, sacc[j][0]);
          sacc[j][1] = fmaf(pj, v1, sacc[j][1]);
        }
      }
#pragma unroll
      for (int j = 0; j < GQ; ++j) {
        pv[(tq * GQ + j) * D + 2 * dp] = sacc[j][0];
        pv[(tq * GQ + j) * D + 2 * dp + 1] = sacc[j][1];
      }
    }
    half_sync(2);
#pragma unroll
    for (int n = 0; n < NACC; ++n) {
      const int it = ht + n * kFastHalf, j = it >> 6, dp = it & 63;
      float s0 = 0.f, s1 = 0.f;
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        s0 += pv[(q4 * GQ + j) * D + 2 * dp];
        s1 += pv[(q4 * GQ + j) * D + 2 * dp + 1];
      }
      accr[n][0] = accr[n][0] * alpha[j] + s0;
      accr[n][1] = accr[n][1] * alpha[j] + s1;
    }
    half_sync(2);   // buffer bi % 2, the logits and the partial sums are free again
    if (bi + 2 < nblk) stage_block(bi + 2);
  }
  cp_async_wait_all();
  float* rec = sc.tail_part + (size_t)u * g.tail_stride;
  if (ht < GQ) {
    rec[ht] = mrun[ht];
    rec[GQ + ht] = lrun[ht];
  }
#pragma unroll
  for (int n = 0; n < NACC; ++n) {
    const int it = ht + n * kFastHalf, j = it >> 6, dp = it & 63;
    rec[2 * GQ + j * D + 2 * dp] = accr[n][0];
    rec[2 * GQ + j * D + 2 * dp + 1] = accr[n][1];
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

template <int R, int GQ>
cudaError_t launch_select_fast(const Geom& g, const CacheBuffers& cb, const Scratch& sc, const void* q,
                               float* scores_out, int32_t* sel_out, int tc_q_mode, bool tail,
                               cudaStream_t s) {
  const size_t smem = FastSmem<R, GQ>::bytes(g.nC);
  auto k = select_fast_kernel<R, GQ>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  k<<<g.U, kFastThreads, smem, s>>>(g, cb, sc, static_cast<const __nv_bfloat16*>(q), scores_out, sel_out,
                                    tc_q_mode, tail ? 1 : 0);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_select(const Geom& g, const CacheBuffers& cb, const Scratch& sc, int dtype,
                          const void* q, float* scores_out, int32_t* sel_out, int tc_q_mode,
                          bool tail, cudaStream_t s) {
  if (dtype == LOWRAM_BF16 && g.d == 128 && g.nC <= kRankMax && (reinterpret_cast<uintptr_t>(q) & 15) == 0) {
#define LOWRAM_SELECT_FAST(RR, GG) \
    if (g.r == RR && g.g == GG) return launch_select_fast<RR, GG>(g, cb, sc, q, scores_out, sel_out, tc_q_mode, tail, s);
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
