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
#include "tc_ptx.cuh"
#include "warp_mma.cuh"

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
// The same computation for the common shapes (bf16, d = 128, r in {64, 128}, g in {4, 8}, at
// most 1024 chunks), as two CTAs of 4 warps per unit: the chunk selection and the raw tail's
// partial softmax do not depend on each other.  Their small dense products run as warp MMAs
// (mma.sync, bf16 in, fp32 accumulation) on rows staged into padded shared memory by cp.async:
// the query projection B_l q_j (exact bf16 inputs), the chunk scores summary . qsum (qsum, an
// fp32 vector, split into bf16 hi + lo columns: ~16 significant bits), the tail logits K q^T
// and the tail sums P V (P split the same way).  The summary rows come in passes of 128
// through two buffers, the second first holding the basis.  The top-k needs no block barrier:
// one warp holds every chunk's order key (nC / 32 per lane) and finds the k-th largest by a
// bitwise binary search with warp-wide counts, then takes the keys equal to it in ascending
// chunk id.
constexpr int kSplitThreads = 128;
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

// dot(8 bf16, 8 consecutive floats of x)
__device__ __forceinline__ float dot8(const uint4& w, const float* x, float a) {
  float v[8];
  bf16x8_to_f32(w, v);
  const float4 q0 = *reinterpret_cast<const float4*>(x);
  const float4 q1 = *reinterpret_cast<const float4*>(x + 4);
  a = fmaf(v[0], q0.x, fmaf(v[1], q0.y, fmaf(v[2], q0.z, fmaf(v[3], q0.w, a))));
  return fmaf(v[4], q1.x, fmaf(v[5], q1.y, fmaf(v[6], q1.z, fmaf(v[7], q1.w, a))));
}

// Shared-memory layout of the fast kernel (byte offsets).  Rows staged from global memory
// (basis, summaries, tail keys and values) are 16-byte-chunk swizzled: chunk c of row r sits
// at chunk (c & ~7) | ((c ^ r) & 7), so the 8 rows an ldmatrix reads start in 8 different bank
// groups without padding.  The small operands built in the kernel are padded rows instead.
template <int R, int GQ>
struct MmaSmem {
  static constexpr int PAD = 136;                         // padded small-operand row, bf16
  static constexpr int PASS = 128;                        // summary rows per staged pass
  static constexpr size_t QB = 0;                         // bf16 [8][PAD]: the unit's queries (rows >= GQ zero)
  // selection CTA
  static constexpr size_t QS = QB + 8 * PAD * 2;          // bf16 [8][PAD]: qsum hi, lo (rows >= 2 zero)
  static constexpr size_t SCORE = QS + 8 * PAD * 2;       // float [1024]: chunk scores by slot, then by id
  // tail CTA (over the selection CTA's QS / SCORE)
  static constexpr size_t PB = QS;                        // bf16 [16][PAD]: probabilities hi / lo
  static constexpr size_t MISC = PB + 16 * PAD * 2;       // float [2][4][GQ]: block maxima, sums
  static constexpr size_t BUF0 = (SCORE + 1024 * 4 + 127) / 128 * 128;   // 32 KB of staged rows
  static constexpr size_t BUF1 = BUF0 + 32768;                           // 32 KB of staged rows
  static constexpr size_t BYTES = BUF1 + 32768;
  static_assert(MISC + 2 * 4 * GQ * 4 <= BUF0, "tail scratch overlaps the staged rows");
};

// Byte offset of 16-byte chunk c of row r in a swizzled block of rows of row_bytes.
__device__ __forceinline__ uint32_t swz(int r, int c, int row_bytes) {
  return (uint32_t)(r * row_bytes + (((c & 7) ^ (r & 7)) | (c & ~7)) * 16);
}

// CTA 2u (or u without a tail) selects for unit u, CTA 2u + 1 runs u's raw tail.
template <int R, int GQ, int NPL>
__global__ void __launch_bounds__(kSplitThreads, 3)
select_mma_kernel(Geom g, CacheBuffers cb, Scratch sc, const __nv_bfloat16* __restrict__ q,
                  float* __restrict__ scores_out, int32_t* __restrict__ sel_out, int tc_q_mode,
                  int do_tail, SelCand cand) {
  constexpr int D = 128;
  using SM = MmaSmem<R, GQ>;
  constexpr int PAD = SM::PAD;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  __nv_bfloat16* qb = reinterpret_cast<__nv_bfloat16*>(smem_raw + SM::QB);
  unsigned char* buf[2] = {smem_raw + SM::BUF0, smem_raw + SM::BUF1};
  const int u = do_tail ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const bool tail_cta = do_tail && (blockIdx.x & 1);
  const Unit un = unit_of(g, u);
  const int l = g.layer0 + un.li;
  const int grp = l / g.G;
  const int NG = g.L / g.G;
  const int nC = g.nC;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gq = lane >> 2, cq = (lane & 3) * 2;   // MMA fragment row / column base
  tc::grid_dep_launch();   // the chunk-attention kernel may start its set-up as SMs free up
  const size_t qoff = ((size_t)(un.li * g.B + un.b) * g.Hq + (size_t)un.hkv * GQ) * D;
  // rows of `rows` x `width` bf16 elements (width % 64 == 0) from global into swizzled rows
  auto stage = [&](unsigned char* dst, const __nv_bfloat16* src, int rows, int width) {
    const int pieces = width / 8;
    for (int it = tid; it < rows * pieces; it += kSplitThreads) {
      const int r = it / pieces, pc = it % pieces;
      cp_async16(dst + swz(r, pc, width * 2), src + (size_t)r * width + pc * 8, true);
    }
    cp_async_commit();
  };
  // the unit's queries as bf16 B-operand rows (exact: the queries are bf16)
  auto load_q = [&]() {
    for (int it = tid; it < 8 * 16; it += kSplitThreads) {
      const int j = it >> 4, pc = it & 15;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (j < GQ) v = __ldg(reinterpret_cast<const uint4*>(q + qoff + (size_t)j * D) + pc);
      *reinterpret_cast<uint4*>(qb + j * PAD + pc * 8) = v;
    }
  };

  if (!tail_cta) {
    // ============================================================ chunk selection
    __nv_bfloat16* qs = reinterpret_cast<__nv_bfloat16*>(smem_raw + SM::QS);
    float* score = reinterpret_cast<float*>(smem_raw + SM::SCORE);
    const __nv_bfloat16* summ = reinterpret_cast<const __nv_bfloat16*>(cb.summary) +
                                (((size_t)un.b * NG + grp) * g.Hkv + un.hkv) * (size_t)g.nLs * R;
    const int n_pass = (g.nL + SM::PASS - 1) / SM::PASS;
    auto stage_pass = [&](int p) {
      stage(buf[p & 1], summ + (size_t)p * SM::PASS * R, min(SM::PASS, g.nL - p * SM::PASS), R);
    };
    // basis rows into buf[1], the first summary pass into buf[0]
    stage(buf[1], reinterpret_cast<const __nv_bfloat16*>(cb.basis) + ((size_t)l * g.Hkv + un.hkv) * R * D, R, D);
    stage_pass(0);
    load_q();
    for (int it = tid; it < 6 * PAD / 8; it += kSplitThreads)   // rows 2..7 of the qsum operand stay zero
      *reinterpret_cast<uint4*>(qs + 2 * PAD + it * 8) = make_uint4(0, 0, 0, 0);
    asm volatile("cp.async.wait_group 1;" ::: "memory");   // the basis
    __syncthreads();
    // --- qt[i][j] = sum_e B_l[i][e] q_j[e]: M = R basis rows, N = 8 (heads), K = 128; warp w
    // takes row tiles w, w + 4, ...
    for (int mt = warp; mt < R / 16; mt += 4) {
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        uint32_t a[4], b[2];
        wm::ldsm_x4(a, buf[1] + swz(16 * mt + (lane & 15), 2 * ks + (lane >> 4), D * 2));
        wm::ldsm_x2(b, qb + (lane & 7) * PAD + ks * 16 + ((lane >> 3) & 1) * 8);
        wm::mma_bf16(acc, a, b);
      }
      // acc: (row i = 16 mt + gq [+ 8], heads cq, cq + 1)
#pragma unroll
      for (int h8 = 0; h8 < 2; ++h8) {
        const int i = 16 * mt + gq + 8 * h8;
        const float v0 = acc[2 * h8], v1 = acc[2 * h8 + 1];
        float part = (cq < GQ ? v0 : 0.f) + (cq + 1 < GQ ? v1 : 0.f);
        part += __shfl_xor_sync(0xffffffffu, part, 1);
        part += __shfl_xor_sync(0xffffffffu, part, 2);
        if ((lane & 3) == 0) {   // qsum[i] as bf16 hi / lo rows of the score operand
          __nv_bfloat16 hi, lo;
          wm::split_bf16(part, hi, lo);
          qs[i] = hi;
          qs[PAD + i] = lo;
        }
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          const int j = cq + x;
          if (j < GQ) {
            const float v = (x ? v1 : v0) * g.qk_scale_log2;
            sc.qt[((size_t)u * GQ + j) * R + i] = v;
            // rows >= GQ of the 16-row copy stay zero (cleared when the scratch is created)
            if (tc_q_mode == 1)
              reinterpret_cast<__nv_bfloat16*>(sc.qt_tc)[((size_t)u * 16 + j) * R + i] = __float2bfloat16_rn(v);
            else if (tc_q_mode == 2)
              reinterpret_cast<__half*>(sc.qt_tc)[((size_t)u * 16 + j) * R + i] = __float2half_rn(v);
          }
        }
      }
    }
    __syncthreads();   // buf[1] (the basis) is free; qsum is complete
    if (n_pass > 1) stage_pass(1);
    // --- scores by live slot, pass by pass: S[c] = summary[c] . (qsum hi + qsum lo)
    const float inv_sqrt_d = rsqrtf((float)D);
    for (int p = 0; p < n_pass; ++p) {
      if (p + 1 < n_pass) asm volatile("cp.async.wait_group 1;" ::: "memory");
      else asm volatile("cp.async.wait_group 0;" ::: "memory");
      __syncthreads();
      const int rows = min(SM::PASS, g.nL - p * SM::PASS);
      const unsigned char* sb = buf[p & 1];
      for (int mt = warp; mt * 16 < rows; mt += 4) {
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ks = 0; ks < R / 16; ++ks) {
          uint32_t a[4], b[2];
          // rows past the pass's last hold stale data: their results are not stored
          wm::ldsm_x4(a, sb + swz(16 * mt + (lane & 15), 2 * ks + (lane >> 4), R * 2));
          wm::ldsm_x2(b, qs + (lane & 7) * PAD + ks * 16 + ((lane >> 3) & 1) * 8);
          wm::mma_bf16(acc, a, b);
        }
        if ((lane & 3) == 0) {   // columns 0, 1 = the hi and lo parts
          const int r0 = p * SM::PASS + 16 * mt + gq;
          if (16 * mt + gq < rows) score[r0] = (acc[0] + acc[1]) * inv_sqrt_d;
          if (16 * mt + gq + 8 < rows) score[r0 + 8] = (acc[2] + acc[3]) * inv_sqrt_d;
        }
      }
      __syncthreads();   // buf[p & 1] is free
      if (p + 2 < n_pass) stage_pass(p + 2);
    }
    // scores by chunk id (evicted chunks -inf); written in place from the top, since slot <= id
    const int16_t* slot = cb.slot ? cb.slot + (((size_t)un.b * NG + grp) * g.Hkv + un.hkv) * g.nCs : nullptr;
    float* so = scores_out ? scores_out + ((size_t)(un.li * g.B + un.b) * g.Hkv + un.hkv) * nC : nullptr;
    float sv[NPL * 32 / kSplitThreads];
#pragma unroll
    for (int x = 0; x < NPL * 32 / kSplitThreads; ++x) {
      const int c = tid + x * kSplitThreads;
      float v = -INFINITY;
      if (c < nC) {
        const int sl = slot ? (int)slot[c] : c;
        if (sl >= 0 && sl < g.nL) v = score[sl];
        else if (sl >= g.nL) atomicOr(sc.err, ERR_SLOT);
        if (so) so[c] = v;
      }
      sv[x] = v;
    }
    __syncthreads();
#pragma unroll
    for (int x = 0; x < NPL * 32 / kSplitThreads; ++x) score[tid + x * kSplitThreads] = sv[x];
    __syncthreads();
    if (warp != 0) return;

    // --- top-k (one warp): lane holds chunks lane*NPL .. lane*NPL + NPL-1; the order key
    // of a score is monotone in the score, and ids >= nC get key 0 (below every chunk's)
    uint32_t key[NPL];
#pragma unroll
    for (int x = 0; x < NPL; x += 4) {
      const float4 f = *reinterpret_cast<const float4*>(&score[lane * NPL + x]);
      const float fv[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
      for (int y = 0; y < 4; ++y) key[x + y] = lane * NPL + x + y < nC ? float_order(fv[y]) : 0u;
    }
    // the k-th largest key: the largest T with #{key >= T} >= k, bit by bit from the top
    uint32_t T = 0;
#pragma unroll 1
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t trial = T | (1u << bit);
      int cnt = 0;
#pragma unroll
      for (int x = 0; x < NPL; ++x) cnt += key[x] >= trial ? 1 : 0;
      if (__reduce_add_sync(0xffffffffu, cnt) >= g.k) T = trial;
    }
    int gt = 0, eq = 0;
#pragma unroll
    for (int x = 0; x < NPL; ++x) {
      gt += key[x] > T ? 1 : 0;
      eq += key[x] == T ? 1 : 0;
    }
    const int need_eq = g.k - (int)__reduce_add_sync(0xffffffffu, gt);   // >= 1 keys equal to T, lowest ids
    int eq_rank = warp_excl_scan(eq);
    uint32_t take = 0;
#pragma unroll
    for (int x = 0; x < NPL; ++x) {
      if (key[x] > T) {
        take |= 1u << x;
      } else if (key[x] == T) {
        if (eq_rank < need_eq) take |= 1u << x;
        ++eq_rank;
      }
    }
    int pos = warp_excl_scan(__popc(take));
    int32_t* sel_slot = sc.sel_slot + (size_t)u * g.k;
    int32_t* sel_id = sc.sel_id + (size_t)u * g.k;
    const size_t ui = (size_t)(un.li * g.B + un.b) * g.Hkv + un.hkv;   // the caller's unit index
    int32_t* sel_user = sel_out ? sel_out + ui * g.k : nullptr;
#pragma unroll
    for (int x = 0; x < NPL; ++x) {
      if (take & (1u << x)) {
        const int c = lane * NPL + x;
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
            cand.score[ui * g.k + pos] = score[c];
            cand.id[ui * g.k + pos] = c + cand.offset;
          }
        }
        ++pos;
      }
    }
    return;
  }

  // ============================================================ raw tail
  // Blocks of 128 tokens staged in shared memory: logits L = K q^T (M = tokens, N = heads),
  // online softmax per head, then acc += P V with P as bf16 hi / lo rows (M = 16) and V read
  // transposed (N = 128 dimensions, K = tokens); the accumulators stay in registers.
  __nv_bfloat16* pb = reinterpret_cast<__nv_bfloat16*>(smem_raw + SM::PB);
  float (*red)[4][GQ] = reinterpret_cast<float (*)[4][GQ]>(smem_raw + SM::MISC);
  int tl = cb.tail_len[un.b];
  if (tl < 0 || tl > g.T) {
    if (tid == 0) atomicOr(sc.err, ERR_TAIL_LEN);
    tl = tl < 0 ? 0 : g.T;
  }
  const size_t toff = (((size_t)un.b * g.L + l) * g.Hkv + un.hkv) * (size_t)g.T * D;
  const __nv_bfloat16* tk = reinterpret_cast<const __nv_bfloat16*>(cb.tail_k) + toff;
  const __nv_bfloat16* tv = reinterpret_cast<const __nv_bfloat16*>(cb.tail_v) + toff;
  auto stage_block = [&](int t0) {   // rows t0 .. t0+127 of K and V, zeros past the tail
    for (int it = tid; it < 128 * 16; it += kSplitThreads) {
      const int r = it >> 4, pc = it & 15;
      const bool in = t0 + r < tl;
      cp_async16(buf[0] + swz(r, pc, D * 2), in ? tk + (size_t)(t0 + r) * D + pc * 8 : tk, in);
      cp_async16(buf[1] + swz(r, pc, D * 2), in ? tv + (size_t)(t0 + r) * D + pc * 8 : tv, in);
    }
    cp_async_commit();
  };
  if (tl > 0) stage_block(0);
  load_q();
  for (int it = tid; it < 16 * PAD / 8; it += kSplitThreads)   // P rows past the heads' stay zero
    *reinterpret_cast<uint4*>(pb + it * 8) = make_uint4(0, 0, 0, 0);
  float m_run[GQ], l_run[GQ];
#pragma unroll
  for (int j = 0; j < GQ; ++j) {
    m_run[j] = -INFINITY;
    l_run[j] = 0.f;
  }
  float acc[4][4];   // P V: warp w holds dimensions 32 w .. 32 w + 31 (n-tiles 4w .. 4w + 3)
#pragma unroll
  for (int nt = 0; nt < 4; ++nt)
#pragma unroll
    for (int x = 0; x < 4; ++x) acc[nt][x] = 0.f;
#pragma unroll 1
  for (int t0 = 0; t0 < tl; t0 += kSelTB) {
    const int nb = min(kSelTB, tl - t0);
    cp_async_wait_all();
    __syncthreads();
    // logits of tokens 32 w .. 32 w + 31 (two m-tiles), heads cq, cq + 1
    float lg[2][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
#pragma unroll
      for (int x = 0; x < 4; ++x) lg[mt][x] = 0.f;
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        uint32_t a[4], b[2];
        wm::ldsm_x4(a, buf[0] + swz(32 * warp + 16 * mt + (lane & 15), 2 * ks + (lane >> 4), D * 2));
        wm::ldsm_x2(b, qb + (lane & 7) * PAD + ks * 16 + ((lane >> 3) & 1) * 8);
        wm::mma_bf16(lg[mt], a, b);
      }
    }
    // per head (column): the block's max over this warp's tokens, then over the warps
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        const int t = 32 * warp + 16 * mt + gq + 8 * (x >> 1);
        lg[mt][x] = t < nb ? lg[mt][x] * g.qk_scale_log2 : -INFINITY;
        mx[x & 1] = fmaxf(mx[x & 1], lg[mt][x]);
      }
#pragma unroll
    for (int x = 0; x < 2; ++x) {
      mx[x] = fmaxf(mx[x], __shfl_xor_sync(0xffffffffu, mx[x], 4));
      mx[x] = fmaxf(mx[x], __shfl_xor_sync(0xffffffffu, mx[x], 8));
      mx[x] = fmaxf(mx[x], __shfl_xor_sync(0xffffffffu, mx[x], 16));
      if (gq == 0 && cq + x < GQ) red[0][warp][cq + x] = mx[x];
    }
    __syncthreads();
    float mnew[2], ps[2] = {0.f, 0.f};
#pragma unroll
    for (int x = 0; x < 2; ++x) {
      const int j = cq + x;
      const float mb = j < GQ ? fmaxf(fmaxf(red[0][0][j], red[0][1][j]), fmaxf(red[0][2][j], red[0][3][j])) : 0.f;
      mnew[x] = j < GQ ? fmaxf(m_run[j], mb) : 0.f;
    }
    // probabilities as bf16 hi / lo rows of the A operand: rows 0 .. GQ-1 hi, GQ .. 2 GQ - 1 lo
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        const int j = cq + (x & 1);
        const int t = 32 * warp + 16 * mt + gq + 8 * (x >> 1);
        if (j < GQ) {
          const float pv = exp2f(lg[mt][x] - mnew[x & 1]);   // 0 past the tail
          ps[x & 1] += pv;
          __nv_bfloat16 hi, lo;
          wm::split_bf16(pv, hi, lo);
          pb[j * PAD + t] = hi;
          pb[(GQ + j) * PAD + t] = lo;
        }
      }
#pragma unroll
    for (int x = 0; x < 2; ++x) {
      ps[x] += __shfl_xor_sync(0xffffffffu, ps[x], 4);
      ps[x] += __shfl_xor_sync(0xffffffffu, ps[x], 8);
      ps[x] += __shfl_xor_sync(0xffffffffu, ps[x], 16);
      if (gq == 0 && cq + x < GQ) red[1][warp][cq + x] = ps[x];
    }
    __syncthreads();
    // rescale the running sums per head, then acc += P V over the block
    float alpha[GQ];
#pragma unroll
    for (int j = 0; j < GQ; ++j) {
      const float mb = fmaxf(fmaxf(red[0][0][j], red[0][1][j]), fmaxf(red[0][2][j], red[0][3][j]));
      const float mn = fmaxf(m_run[j], mb);
      alpha[j] = exp2f(m_run[j] - mn);   // 0 while m_run = -inf
      l_run[j] = l_run[j] * alpha[j] + (red[1][0][j] + red[1][1][j]) + (red[1][2][j] + red[1][3][j]);
      m_run[j] = mn;
    }
    // accumulator rows: gq (c0, c1) and gq + 8 (c2, c3) of the 16 P rows; row r's head is r % GQ
    // when r < 2 GQ (its hi or lo part), none otherwise
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      const float a0 = gq < 2 * GQ ? alpha[gq % GQ] : 0.f;
      const float a1 = gq + 8 < 2 * GQ ? alpha[(gq + 8) % GQ] : 0.f;
      acc[nt][0] *= a0;
      acc[nt][1] *= a0;
      acc[nt][2] *= a1;
      acc[nt][3] *= a1;
    }
#pragma unroll
    for (int ks = 0; ks < kSelTB / 16; ++ks) {
      uint32_t a[4];
      wm::ldsm_x4(a, pb + (lane & 15) * PAD + ks * 16 + (lane >> 4) * 8);
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        uint32_t b[2];
        // B = V[token][dim]: k = token rows, n = dims, read transposed
        wm::ldsm_x2_t(b, buf[1] + swz(ks * 16 + (lane & 15), 4 * warp + nt, D * 2));
        wm::mma_bf16(acc[nt], a, b);
      }
    }
    if (t0 + kSelTB < tl) {   // every thread is done with this block's rows
      __syncthreads();
      stage_block(t0 + kSelTB);
    }
  }
  // the tail record (log2-domain max, sum, sums per head): hi and lo rows of head j are rows j
  // and GQ + j of the accumulator
  float* rec = sc.tail_part + (size_t)u * g.tail_stride;
  if (GQ == 8) {
    // rows gq (hi) and gq + 8 (lo) of the same lane
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      const int dd = 32 * warp + 8 * nt + cq;
      rec[2 * GQ + gq * D + dd] = acc[nt][0] + acc[nt][2];
      rec[2 * GQ + gq * D + dd + 1] = acc[nt][1] + acc[nt][3];
    }
  } else {
    // GQ = 4: hi rows 0-3 in lanes 0-15, lo rows 4-7 in lanes 16-31 (c0, c1)
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      const float o0 = acc[nt][0] + __shfl_xor_sync(0xffffffffu, acc[nt][0], 16);
      const float o1 = acc[nt][1] + __shfl_xor_sync(0xffffffffu, acc[nt][1], 16);
      if (gq < GQ) {
        const int dd = 32 * warp + 8 * nt + cq;
        rec[2 * GQ + gq * D + dd] = o0;
        rec[2 * GQ + gq * D + dd + 1] = o1;
      }
    }
  }
  if (tid < GQ) {
    rec[tid] = m_run[tid];
    rec[GQ + tid] = l_run[tid];
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
cudaError_t launch_select_split(const Geom& g, const CacheBuffers& cb, const Scratch& sc, const void* q,
                                float* scores_out, int32_t* sel_out, int tc_q_mode, bool tail, cudaStream_t s,
                                SelCand cand) {
  using SM = MmaSmem<R, GQ>;
  const size_t smem = SM::BYTES;
  auto k = select_mma_kernel<R, GQ, NPL>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)g.U * (tail ? 2u : 1u);
  k<<<grid, kSplitThreads, smem, s>>>(g, cb, sc, static_cast<const __nv_bfloat16*>(q), scores_out, sel_out,
                                       tc_q_mode, tail ? 1 : 0, cand);
  return cudaGetLastError();
}

template <int R, int GQ>
cudaError_t launch_select_fast(const Geom& g, const CacheBuffers& cb, const Scratch& sc, const void* q,
                               float* scores_out, int32_t* sel_out, int tc_q_mode, bool tail, cudaStream_t s,
                               SelCand cand) {
  if (g.nC <= 256) return launch_select_split<R, GQ, 8>(g, cb, sc, q, scores_out, sel_out, tc_q_mode, tail, s, cand);
  if (g.nC <= 512) return launch_select_split<R, GQ, 16>(g, cb, sc, q, scores_out, sel_out, tc_q_mode, tail, s, cand);
  return launch_select_split<R, GQ, 32>(g, cb, sc, q, scores_out, sel_out, tc_q_mode, tail, s, cand);
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
