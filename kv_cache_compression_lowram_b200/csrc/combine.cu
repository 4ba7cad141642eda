// Final step: merge the softmax partials of a unit (raw tail + every chunk piece),
// apply the predictor's second layer once to the softmax-weighted hidden sum and
// normalise:
//     o_j = (W2 . sum_t p_jt h_t + sum_t p_jt delta_t + sum_tail p_jt v_t) / sum_t p_jt
// This is the exact regrouping of sum_t p_jt (W2 h_t + delta_t) for the rebuilt values of
// "LowRAM Compresses KV Cache Asymmetrically", section "Core Mechanism" (Vhat = f(K) plus
// delta for the worst tokens), inside the attention of "OjaKV", section 3.
// Also: the create-time fold W1' = W1 B_l^T and the device-side table check.
#include "lowram_internal.cuh"
#include "warp_mma.cuh"
#include "reuse.cuh"

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

// The same merge for bf16 with d = 128, h = 256, g in {4, 8}: one CTA for up to 16 / g units
// of one (layer, KV head), so W2 is read once for all of them and its product with their 16
// merged hidden-sum vectors runs as warp MMAs (mma.sync, fp32 accumulation; each fp32 sum is
// split into bf16 hi + lo columns so the product keeps fp32-level accuracy).  W2 streams into
// padded shared memory (rows 528 bytes apart: conflict-free ldmatrix) while the pieces are
// merged.  Up to kCombPieces pieces per unit; more take the generic kernel.
constexpr int kCombPieces = 8;
constexpr int kCombThreads = 256;

template <int GQ, bool LIST = false>
struct CombSmem {
  static constexpr int UB = 16 / GQ;          // units per CTA
  static constexpr int NR = UB * GQ;          // (unit, head) rows: 16
  static constexpr int WROW = 256 + 8;        // padded row, bf16 elements
  static constexpr size_t W2 = 0;                                   // bf16 [128][WROW]
  static constexpr size_t BM = W2 + 128 * WROW * 2;                 // bf16 [2 NR][WROW]: hi, lo rows
  static constexpr size_t ACCD = BM + 2 * NR * WROW * 2;            // float [NR][128]
  static constexpr int MAXP = LIST ? 33 : kCombPieces;             // pieces per unit
  static constexpr size_t WT = ACCD + NR * 128 * 4;                 // float [NR][MAXP + 2]
  static constexpr size_t LS = WT + NR * (MAXP + 2) * 4;            // float [NR]
  static constexpr size_t MS = LS + NR * 4;                         // float [NR]: merged max
  static constexpr size_t PC = MS + NR * 4;                         // int [UB][2]: first piece, pieces
  static constexpr size_t BYTES = PC + UB * 2 * 4;
};

__device__ __forceinline__ void cp_async16c(void* smem_dst, const void* gsrc) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst))),
               "l"(gsrc)
               : "memory");
}

// LIST: the pieces come from an explicit tile list (sc.tile_ptr / sc.tile_total; units may
// have any number of tiles, none included) and, when extra_rec is given, every unit has one
// extra record in the tail's format (extra_rec, [U][tail_stride]), merged like the tail.
// PART: the output is left unnormalised, one fp32 row [m (log2 units), l, y[0..d)] per
// (layer, sequence, query head) in `part` (a context shard's partial), instead of bf16 o.
template <int GQ, bool LIST, bool PART = false>
__global__ void __launch_bounds__(kCombThreads, 2)
combine_mma_kernel(Geom g, CacheBuffers cb, Scratch sc, const float* __restrict__ extra_rec,
                   __nv_bfloat16* __restrict__ out, float* __restrict__ part) {
  constexpr int D = 128, H = 256;
  using SM = CombSmem<GQ, LIST>;
  constexpr int UB = SM::UB, NR = SM::NR, WROW = SM::WROW, MAXP = SM::MAXP;
  extern __shared__ __align__(128) unsigned char smem[];
  __nv_bfloat16* w2s = reinterpret_cast<__nv_bfloat16*>(smem + SM::W2);
  __nv_bfloat16* bms = reinterpret_cast<__nv_bfloat16*>(smem + SM::BM);
  float (*accd)[D] = reinterpret_cast<float (*)[D]>(smem + SM::ACCD);
  float (*wt)[MAXP + 2] = reinterpret_cast<float (*)[MAXP + 2]>(smem + SM::WT);
  float* ls = reinterpret_cast<float*>(smem + SM::LS);
  float* ms = reinterpret_cast<float*>(smem + SM::MS);
  const bool has_x = LIST && extra_rec != nullptr;
  int (*pc)[2] = reinterpret_cast<int (*)[2]>(smem + SM::PC);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nbb = (g.B + UB - 1) / UB;
  const int pair = blockIdx.x / nbb;              // li * Hkv + hkv
  const int b0 = (blockIdx.x % nbb) * UB;
  const int nb = min(UB, g.B - b0);
  const int li = pair / g.Hkv, hkv = pair % g.Hkv;
  const int l = g.layer0 + li;
  const int u0 = pair * g.B + b0;                 // units u0 .. u0 + nb - 1
  // W2 of (l, hkv) into padded rows, asynchronously: 128 rows x 32 pieces of 16 bytes
  const __nv_bfloat16* w2 = reinterpret_cast<const __nv_bfloat16*>(cb.w2) + ((size_t)l * g.Hkv + hkv) * D * H;
#pragma unroll 4
  for (int x = 0; x < D * H / 8 / kCombThreads; ++x) {
    const int it = tid + x * kCombThreads, row = it >> 5, piece = it & 31;
    cp_async16c(w2s + row * WROW + piece * 8, w2 + (size_t)row * H + piece * 8);
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
  // W2 streams in while the chunk-attention kernel finishes (programmatic dependent launch);
  // its partial records are read only after this
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // merge weights of every (unit, head) row: w_r = 2^(m_r - M) over the unit's pieces and tail
  const long long total = LIST ? (long long)*sc.tile_total : (long long)g.U * g.k;
  if (tid < NR) {
    const int r = tid, bi = r / GQ, j = r % GQ;
    float L = 0.f;
    if (bi < nb) {
      const int u = u0 + bi;
      int c0 = 0, nrec = 0;
      if (LIST) {
        const int p0 = sc.tile_ptr[u], p1 = sc.tile_ptr[u + 1];
        if (p1 > p0) {
          c0 = cta_of_tile(total, g.P, p0);
          nrec = cta_of_tile(total, g.P, p1 - 1) - c0 + 1;
        }
      } else {
        c0 = cta_of_tile(total, g.P, (long long)u * g.k);
        nrec = cta_of_tile(total, g.P, (long long)(u + 1) * g.k - 1) - c0 + 1;
      }
      if (j == 0) {
        pc[bi][0] = c0;
        pc[bi][1] = nrec;
        if (nrec > MAXP || (!LIST && nrec > g.max_rec)) atomicOr(sc.err, ERR_SELECT);   // cannot happen
      }
      const int np = min(nrec, MAXP);
      const float* trec = sc.tail_part + (size_t)u * g.tail_stride;
      const float* xrec = has_x ? extra_rec + (size_t)u * g.tail_stride : trec;
      float M = trec[j];
      if (has_x) M = fmaxf(M, xrec[j]);
      for (int p = 0; p < np; ++p) M = fmaxf(M, sc.part[(size_t)(u + c0 + p) * g.rec_stride + j]);
      for (int p = 0; p < np; ++p) {
        const float* rec = sc.part + (size_t)(u + c0 + p) * g.rec_stride;
        const float w = rec[j] == -INFINITY ? 0.f : exp2f(rec[j] - M);
        wt[r][p] = w;
        L = fmaf(w, rec[GQ + j], L);
      }
      const float w_t = trec[j] == -INFINITY ? 0.f : exp2f(trec[j] - M);
      wt[r][MAXP] = w_t;
      L = fmaf(w_t, trec[GQ + j], L);
      if (has_x) {
        const float w_x = xrec[j] == -INFINITY ? 0.f : exp2f(xrec[j] - M);
        wt[r][MAXP + 1] = w_x;
        L = fmaf(w_x, xrec[GQ + j], L);
      }
      ms[r] = M;
    }
    ls[r] = L;
  }
  __syncthreads();
  // merged hidden sums as bf16 hi / lo rows, merged residual + tail sums: thread = (row r,
  // slice s of 16 hidden units and 8 dimensions)
  {
    const int r = tid >> 4, s = tid & 15, bi = r / GQ, j = r % GQ;
    float hs[16], ds[8];
#pragma unroll
    for (int x = 0; x < 16; ++x) hs[x] = 0.f;
#pragma unroll
    for (int x = 0; x < 8; ++x) ds[x] = 0.f;
    if (bi < nb) {
      const int u = u0 + bi;
      const int c0 = pc[bi][0], np = min(pc[bi][1], MAXP);
      for (int p = 0; p < np; ++p) {
        const float* rec = sc.part + (size_t)(u + c0 + p) * g.rec_stride;
        const float w = wt[r][p];
        const float4* hv = reinterpret_cast<const float4*>(rec + 2 * GQ + j * H + s * 16);
        const float4* dv = reinterpret_cast<const float4*>(rec + 2 * GQ + GQ * H + j * D + s * 8);
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const float4 v = hv[x];
          hs[4 * x] = fmaf(w, v.x, hs[4 * x]);
          hs[4 * x + 1] = fmaf(w, v.y, hs[4 * x + 1]);
          hs[4 * x + 2] = fmaf(w, v.z, hs[4 * x + 2]);
          hs[4 * x + 3] = fmaf(w, v.w, hs[4 * x + 3]);
        }
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          const float4 v = dv[x];
          ds[4 * x] = fmaf(w, v.x, ds[4 * x]);
          ds[4 * x + 1] = fmaf(w, v.y, ds[4 * x + 1]);
          ds[4 * x + 2] = fmaf(w, v.z, ds[4 * x + 2]);
          ds[4 * x + 3] = fmaf(w, v.w, ds[4 * x + 3]);
        }
      }
#pragma unroll
      for (int xr = 0; xr < (LIST ? 2 : 1); ++xr) {   // the tail, then the extra record
        if (xr == 1 && !has_x) break;
        const float w_t = wt[r][MAXP + xr];
        const float* base = xr ? extra_rec : sc.tail_part;
        const float4* tv = reinterpret_cast<const float4*>(base + (size_t)u * g.tail_stride + 2 * GQ + j * D + s * 8);
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          const float4 v = tv[x];
          ds[4 * x] = fmaf(w_t, v.x, ds[4 * x]);
          ds[4 * x + 1] = fmaf(w_t, v.y, ds[4 * x + 1]);
          ds[4 * x + 2] = fmaf(w_t, v.z, ds[4 * x + 2]);
          ds[4 * x + 3] = fmaf(w_t, v.w, ds[4 * x + 3]);
        }
      }
    }
    __nv_bfloat16 hi[16], lo[16];
#pragma unroll
    for (int x = 0; x < 16; ++x) wm::split_bf16(hs[x], hi[x], lo[x]);
    *reinterpret_cast<uint4*>(bms + (2 * r) * WROW + s * 16) = *reinterpret_cast<const uint4*>(hi);
    *reinterpret_cast<uint4*>(bms + (2 * r) * WROW + s * 16 + 8) = *reinterpret_cast<const uint4*>(hi + 8);
    *reinterpret_cast<uint4*>(bms + (2 * r + 1) * WROW + s * 16) = *reinterpret_cast<const uint4*>(lo);
    *reinterpret_cast<uint4*>(bms + (2 * r + 1) * WROW + s * 16 + 8) = *reinterpret_cast<const uint4*>(lo + 8);
#pragma unroll
    for (int x = 0; x < 8; ++x) accd[r][s * 8 + x] = ds[x];
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  __syncthreads();
  // y[d][n] = sum_h W2[d][h] Bm[n][h]: warp w takes dimensions 16w .. 16w+15, all 32 columns
  float acc[4][4];
#pragma unroll
  for (int nt = 0; nt < 4; ++nt)
#pragma unroll
    for (int x = 0; x < 4; ++x) acc[nt][x] = 0.f;
#pragma unroll 4
  for (int ks = 0; ks < H / 16; ++ks) {
    uint32_t a[4];
    wm::ldsm_x4(a, w2s + (16 * warp + (lane & 15)) * WROW + ks * 16 + (lane >> 4) * 8);
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      uint32_t b[2];
      wm::ldsm_x2(b, bms + (8 * nt + (lane & 7)) * WROW + ks * 16 + ((lane >> 3) & 1) * 8);
      wm::mma_bf16(acc[nt], a, b);
    }
  }
  // columns (c, c + 1) of n-tile nt are the hi and lo parts of row r = 4 nt + lane % 4
  const int gq = lane >> 2;
#pragma unroll
  for (int nt = 0; nt < 4; ++nt) {
    const int r = 4 * nt + (lane & 3), bi = r / GQ, j = r % GQ;
    if (bi < nb) {
      const size_t orow = (size_t)(li * g.B + b0 + bi) * g.Hq + (size_t)hkv * GQ + j;
      const int d0 = 16 * warp + gq;
      if (PART) {
        float* pr = part + orow * (D + 2);
        pr[2 + d0] = acc[nt][0] + acc[nt][1] + accd[r][d0];
        pr[2 + d0 + 8] = acc[nt][2] + acc[nt][3] + accd[r][d0 + 8];
        if (warp == 0 && gq == 0) {
          pr[0] = ms[r];
          pr[1] = ls[r];
        }
      } else {
        __nv_bfloat16* o = out + orow * D;
        o[d0] = __float2bfloat16_rn((acc[nt][0] + acc[nt][1] + accd[r][d0]) / ls[r]);
        o[d0 + 8] = __float2bfloat16_rn((acc[nt][2] + acc[nt][3] + accd[r][d0 + 8]) / ls[r]);
      }
    }
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
  } else if (g.d == 128 && g.h == 256 && (g.g == 4 || g.g == 8) && g.max_rec <= kCombPieces) {
    auto k = g.g == 4 ? combine_mma_kernel<4, false> : combine_mma_kernel<8, false>;
    const size_t sm = g.g == 4 ? CombSmem<4>::BYTES : CombSmem<8>::BYTES;
    const int ub = 16 / g.g;
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t lc = {};
    lc.gridDim = dim3((unsigned)(g.n_layers * g.Hkv) * (unsigned)((g.B + ub - 1) / ub));
    lc.blockDim = dim3(kCombThreads);
    lc.dynamicSmemBytes = sm;
    lc.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    lc.attrs = at;
    lc.numAttrs = 1;
    e = cudaLaunchKernelEx(&lc, k, g, cb, sc, static_cast<const float*>(nullptr), static_cast<__nv_bfloat16*>(out),
                           static_cast<float*>(nullptr));
    if (e != cudaSuccess) return e;
  } else {
    auto k = combine_kernel<__nv_bfloat16>;
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<g.U, kThreads, smem, s>>>(g, cb, sc, static_cast<__nv_bfloat16*>(out));
  }
  return cudaGetLastError();
}

cudaError_t launch_combine_list(const Geom& g, const CacheBuffers& cb, const Scratch& sc, const float* extra_rec,
                                void* out, cudaStream_t s) {
  if (g.d != 128 || g.h != 256 || !(g.g == 4 || g.g == 8) || g.k > 32) return cudaErrorNotSupported;
  auto k = g.g == 4 ? combine_mma_kernel<4, true> : combine_mma_kernel<8, true>;
  const size_t sm = g.g == 4 ? CombSmem<4, true>::BYTES : CombSmem<8, true>::BYTES;
  const int ub = 16 / g.g;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)(g.n_layers * g.Hkv) * (unsigned)((g.B + ub - 1) / ub);
  k<<<grid, kCombThreads, sm, s>>>(g, cb, sc, extra_rec, static_cast<__nv_bfloat16*>(out), static_cast<float*>(nullptr));
  return cudaGetLastError();
}

cudaError_t launch_combine_partial_fast(const Geom& g, const CacheBuffers& cb, const Scratch& sc, float* partial,
                                        cudaStream_t s) {
  if (g.d != 128 || g.h != 256 || !(g.g == 4 || g.g == 8) || g.k > 32) return cudaErrorNotSupported;
  auto k = g.g == 4 ? combine_mma_kernel<4, true, true> : combine_mma_kernel<8, true, true>;
  const size_t sm = g.g == 4 ? CombSmem<4, true>::BYTES : CombSmem<8, true>::BYTES;
  const int ub = 16 / g.g;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)(g.n_layers * g.Hkv) * (unsigned)((g.B + ub - 1) / ub);
  k<<<grid, kCombThreads, sm, s>>>(g, cb, sc, nullptr, nullptr, partial);
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
