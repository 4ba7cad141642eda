// Prefill-side encoder: dense keys and values -> the compressed cache arrays, with a given
// basis and predictor (no fitting).  "LowRAM Compresses KV Cache Asymmetrically", sections
// "Cross-Layer Low-Rank Key Compression" (keys of a layer group on one basis),
// "Core Mechanism: Predict Values and Keep Difficult Residuals" (Vhat = f(Khat),
// delta = V - Vhat kept for the worst-predicted tokens) and "Composition with Quantization
// and Eviction" (int8 rows).
//
// Kernels, in launch order:
//   fold (combine.cu)   W1' = W1 B_l^T per (layer, KV head), fp32 [r][h]
//   enc_coeff_kernel    per (b, group, KV head, chunk): a = (1/G) sum_l K_l B_l^T (the
//                       least-squares coefficients for bases with orthonormal rows), stored
//                       as bf16 or int8 rows, and the chunk summary (mean stored row)
//   enc_resid_kernel    per (b, layer, KV head, chunk): H = silu(a W1'^T), Vhat = H W2^T,
//                       delta = V - Vhat; pass 1 writes |delta_t|_2, pass 2 the records of
//                       the flagged tokens
//   enc_select_kernel   per (b, layer, KV head): the n_resid largest norms (ties to the
//                       lower token) by a radix select, flags and the CSR offsets
// enc_resid_kernel is the CUDA-core fp32 form (any store); enc_resid_tc_kernel the tcgen05
// form of the same pass for bf16 stores (D1 = W1'/2 . A^T, silu into shared memory as fp16,
// Vhat = W2 . H with W2 in fp16, fp32 accumulators in TMEM).
#include <algorithm>
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "lowram_internal.cuh"
#include "upkeep.cuh"
#include "tc_ptx.cuh"

namespace lowram {
namespace {

constexpr int kEncThreads = 256;
constexpr int kEncD = 128;     // head dim
constexpr int kEncH = 256;     // predictor hidden width
constexpr int kKT = 32;        // contraction tile

__device__ __forceinline__ void load_bf16x8(const __nv_bfloat16* p, float* v) {
  const uint4 w = *reinterpret_cast<const uint4*>(p);
  const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    v[2 * h] = __uint_as_float(ww[h] << 16);
    v[2 * h + 1] = __uint_as_float(ww[h] & 0xffff0000u);
  }
}

__device__ __forceinline__ uint4 pack_bf16x8(const float* v) {
  uint32_t o[4];
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    const __nv_bfloat162 p = __floats2bfloat162_rn(v[2 * h], v[2 * h + 1]);
    o[h] = *reinterpret_cast<const uint32_t*>(&p);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// int8 row encoding shared by coefficients and residual rows: scale = fp16(max|x| / 127),
// code = round-half-even(x / scale) clamped to +-127 (0 for an all-zero row).
__device__ __forceinline__ void quantize8(const float* x, float amax, __half* scale_out, uint2* codes,
                                          float* deq) {
  const __half sh = __float2half_rn(amax / 127.f);
  const float s = __half2float(sh);
  uint32_t w[2] = {0u, 0u};
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    float q = s > 0.f ? rintf(x[j] / s) : 0.f;
    q = fminf(fmaxf(q, -127.f), 127.f);
    if (deq) deq[j] = q * s;
    w[j >> 2] |= ((uint32_t)(int)q & 0xffu) << (8 * (j & 3));
  }
  *codes = make_uint2(w[0], w[1]);
  *scale_out = sh;
}

// The same encoding for a row whose fp16 scale s (> 0 or 0) and reciprocal r are known:
// round-half-even of x / s from a first guess rint(x r), corrected by the exact
// remainder x - q s (an fma: q s has at most 19 significant bits and lies within s of x, so
// the remainder is representable), a tie going to even.  One division per row instead of
// one per value; the result is the rounding of the exact quotient.
__device__ __forceinline__ float rne_quot(float x, float s, float r) {
  float q = rintf(x * r);
  const float rem = fmaf(-q, s, x);
  const float h = 0.5f * s;
  const bool odd = ((int)q & 1) != 0;
  if (rem > h || (rem == h && odd)) q += 1.f;
  else if (rem < -h || (rem == -h && odd)) q -= 1.f;
  return q;
}
// (x r is within 2^-22 relative of x / s, i.e. within 4e-5 for |x / s| <= 127.5, so its
// nearest integer is the answer unless x r lies within 1e-4 of a half-integer; only then is
// the exact remainder consulted.)  The code of one value of a row with scale s and r = 1 / s
// (0 when s = 0), clamped to [-127, 127].
__device__ __forceinline__ uint32_t code8_scaled(float x, float s, float r) {
  const float y = x * r;
  float q = rintf(y);
  if (fabsf(y - q) > 0.4999f) q = rne_quot(x, s, r);
  q = s > 0.f ? fminf(fmaxf(q, -127.f), 127.f) : 0.f;
  return (uint32_t)(int)q & 0xffu;
}

// --------------------------------------------------------------------- coefficients
// Thread (ty, tx): tokens ty*TM .. +TM, ranks tx*8 .. +8.  Per (layer, 32-wide slice of
// d): the chunk's key slice and the basis slice go to shared memory transposed (k-major),
// then every thread accumulates its TM x 8 block.
template <int R, int C, bool I8>
__global__ void __launch_bounds__(kEncThreads)
enc_coeff_kernel(int L, int G, int Hkv, int N, const __nv_bfloat16* __restrict__ keys,
                 const __nv_bfloat16* __restrict__ basis, void* __restrict__ coeff,
                 __half* __restrict__ coeff_scale, __nv_bfloat16* __restrict__ summary) {
  constexpr int TX = R / 8, TY = kEncThreads / TX, TM = C / TY;
  static_assert(TM * TY == C && TM >= 1, "tile shape");
  __shared__ __align__(16) float ks[kKT][C];
  __shared__ __align__(16) float bs[kKT][R];
  __shared__ float red[TY][R];
  const int c = blockIdx.x, hkv = blockIdx.y;
  const int b = blockIdx.z / (L / G), grp = blockIdx.z % (L / G);
  const int tid = threadIdx.x, tx = tid % TX, ty = tid / TX;
  const int nC = N / C;
  float acc[TM][8];
#pragma unroll
  for (int i = 0; i < TM; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

  for (int li = 0; li < G; ++li) {
    const int l = grp * G + li;
    const __nv_bfloat16* krow = keys + ((((size_t)b * L + l) * Hkv + hkv) * N + (size_t)c * C) * kEncD;
    const __nv_bfloat16* brow = basis + (((size_t)l * Hkv + hkv) * R) * kEncD;
    for (int k0 = 0; k0 < kEncD; k0 += kKT) {
      __syncthreads();
      // C rows x 32 columns of keys, R rows x 32 columns of the basis: 8 bf16 per piece
      for (int p = tid; p < C * (kKT / 8); p += kEncThreads) {
        const int t = p / (kKT / 8), e = (p % (kKT / 8)) * 8;
        float v[8];
        load_bf16x8(krow + (size_t)t * kEncD + k0 + e, v);
#pragma unroll
        for (int j = 0; j < 8; ++j) ks[e + j][t] = v[j];
      }
      for (int p = tid; p < R * (kKT / 8); p += kEncThreads) {
        const int rr = p / (kKT / 8), e = (p % (kKT / 8)) * 8;
        float v[8];
        load_bf16x8(brow + (size_t)rr * kEncD + k0 + e, v);
#pragma unroll
        for (int j = 0; j < 8; ++j) bs[e + j][rr] = v[j];
      }
      __syncthreads();
#pragma unroll 4
      for (int k = 0; k < kKT; ++k) {
        float a[TM], bb[8];
#pragma unroll
        for (int i = 0; i < TM; ++i) a[i] = ks[k][ty * TM + i];
#pragma unroll
        for (int j = 0; j < 8; ++j) bb[j] = bs[k][tx * 8 + j];
#pragma unroll
        for (int i = 0; i < TM; ++i)
#pragma unroll
          for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], bb[j], acc[i][j]);
      }
    }
  }

  // store each row; the stored (dequantised) values feed the chunk summary
  const float inv_g = 1.f / (float)G;
  const size_t row0 = (((size_t)b * (L / G) + grp) * Hkv + hkv) * N + (size_t)c * C;
  float colsum[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) colsum[j] = 0.f;
#pragma unroll
  for (int i = 0; i < TM; ++i) {
    const int t = ty * TM + i;
    float x[8], deq[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) x[j] = acc[i][j] * inv_g;
    if (I8) {
      float m = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) m = fmaxf(m, fabsf(x[j]));
#pragma unroll
      for (int o = 1; o < TX; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      __half sh;
      uint2 codes;
      quantize8(x, m, &sh, &codes, deq);
      *reinterpret_cast<uint2*>(static_cast<int8_t*>(coeff) + (row0 + t) * R + tx * 8) = codes;
      if (tx == 0) coeff_scale[row0 + t] = sh;
    } else {
      const uint4 p = pack_bf16x8(x);
      *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(coeff) + (row0 + t) * R + tx * 8) = p;
      const uint32_t pw[4] = {p.x, p.y, p.z, p.w};
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        deq[2 * h] = __uint_as_float(pw[h] << 16);
        deq[2 * h + 1] = __uint_as_float(pw[h] & 0xffff0000u);
      }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) colsum[j] += deq[j];
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) red[ty][tx * 8 + j] = colsum[j];
  __syncthreads();
  for (int rr = tid; rr < R; rr += kEncThreads) {
    float s = 0.f;
    for (int y = 0; y < TY; ++y) s += red[y][rr];
    summary[((((size_t)b * (L / G) + grp) * Hkv + hkv) * nC + c) * R + rr] = __float2bfloat16_rn(s / (float)C);
  }
}

// ------------------------------------------------------------------------ residuals
// Thread (ty, tx): tokens ty*TM .. +TM; hidden units (phase A) or value dims (phase B)
// tx*8 .. +8.  Shared memory: the chunk's stored coefficients (k-major), one half of the
// hidden activations (k-major) and a 32-row weight tile.
template <int R, int C>
struct ResidSmem {
  static constexpr size_t bytes() { return ((size_t)R * C + (size_t)128 * C + (size_t)kKT * 128) * 4 + (size_t)C * 4; }
};

template <int R, int C, bool I8, bool EMIT>
__global__ void __launch_bounds__(kEncThreads, 1)
enc_resid_kernel(int L, int G, int Hkv, int N, int n_res, const void* __restrict__ coeff,
                 const __half* __restrict__ coeff_scale, const float* __restrict__ w1f_t,
                 const __nv_bfloat16* __restrict__ w2, const __nv_bfloat16* __restrict__ values,
                 float* __restrict__ norms, const uint8_t* __restrict__ flags,
                 const int32_t* __restrict__ res_ptr, uint16_t* __restrict__ res_pos, void* __restrict__ res_val,
                 __half* __restrict__ res_scale) {
  constexpr int TX = 16, TY = kEncThreads / TX, TM = C / TY;
  static_assert(TM * TY == C, "tile shape");
  extern __shared__ __align__(16) float esm[];
  float* as = esm;                        // [R][C]   stored coefficients, k-major
  float* hs = as + R * C;                 // [128][C] silu(pre-activations) of one half
  float* ws = hs + 128 * C;               // [32][128] weight tile
  int* fl = reinterpret_cast<int*>(ws + kKT * 128);   // [C] flags (EMIT)
  const int c = blockIdx.x, hkv = blockIdx.y;
  const int b = blockIdx.z / L, l = blockIdx.z % L;
  const int grp = l / G;
  const int tid = threadIdx.x, tx = tid % TX, ty = tid / TX;
  const int nC = N / C;
  const size_t unit = ((size_t)b * L + l) * Hkv + hkv;
  const size_t row0 = (((size_t)b * (L / G) + grp) * Hkv + hkv) * N + (size_t)c * C;

  // the chunk's stored coefficient rows, dequantised, transposed
  for (int p = tid; p < C * (R / 8); p += kEncThreads) {
    const int t = p / (R / 8), e = (p % (R / 8)) * 8;
    float v[8];
    if (I8) {
      const uint2 q = *reinterpret_cast<const uint2*>(static_cast<const int8_t*>(coeff) + (row0 + t) * R + e);
      const float s = __half2float(coeff_scale[row0 + t]);
      const uint32_t qw[2] = {q.x, q.y};
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = (float)(int8_t)((qw[j >> 2] >> (8 * (j & 3))) & 0xffu) * s;
    } else {
      load_bf16x8(static_cast<const __nv_bfloat16*>(coeff) + (row0 + t) * R + e, v);
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) as[(e + j) * C + t] = v[j];
  }
  if (EMIT)
    for (int t = tid; t < C; t += kEncThreads) fl[t] = flags[unit * N + (size_t)c * C + t];

  const float* w1l = w1f_t + ((size_t)l * Hkv + hkv) * R * kEncH;          // [R][256]
  const __nv_bfloat16* w2l = w2 + ((size_t)l * Hkv + hkv) * kEncD * kEncH;  // [128][256]
  float vacc[TM][8];
#pragma unroll
  for (int i = 0; i < TM; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) vacc[i][j] = 0.f;

  for (int hh = 0; hh < 2; ++hh) {
    // phase A: hidden half hh
    float hacc[TM][8];
#pragma unroll
    for (int i = 0; i < TM; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) hacc[i][j] = 0.f;
    for (int k0 = 0; k0 < R; k0 += kKT) {
      __syncthreads();
      for (int p = tid; p < kKT * 128 / 4; p += kEncThreads) {
        const int k = p / 32, j4 = (p % 32) * 4;
        *reinterpret_cast<float4*>(ws + k * 128 + j4) =
            *reinterpret_cast<const float4*>(w1l + (size_t)(k0 + k) * kEncH + hh * 128 + j4);
      }
      __syncthreads();
#pragma unroll 4
      for (int k = 0; k < kKT; ++k) {
        float a[TM], bb[8];
#pragma unroll
        for (int i = 0; i < TM; ++i) a[i] = as[(k0 + k) * C + ty * TM + i];
#pragma unroll
        for (int j = 0; j < 8; ++j) bb[j] = ws[k * 128 + tx * 8 + j];
#pragma unroll
        for (int i = 0; i < TM; ++i)
#pragma unroll
          for (int j = 0; j < 8; ++j) hacc[i][j] = fmaf(a[i], bb[j], hacc[i][j]);
      }
    }
    __syncthreads();   // the previous half's activations are no longer read
#pragma unroll
    for (int i = 0; i < TM; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float x = hacc[i][j];
        hs[(tx * 8 + j) * C + ty * TM + i] = x / (1.f + expf(-x));
      }
    // phase B: value dims += H_half . W2[:, half]^T
    for (int k0 = 0; k0 < 128; k0 += kKT) {
      __syncthreads();
      for (int p = tid; p < 128 * (kKT / 8); p += kEncThreads) {
        const int e = p / (kKT / 8), kk = (p % (kKT / 8)) * 8;
        float v[8];
        load_bf16x8(w2l + (size_t)e * kEncH + hh * 128 + k0 + kk, v);
#pragma unroll
        for (int j = 0; j < 8; ++j) ws[(kk + j) * 128 + e] = v[j];
      }
      __syncthreads();
#pragma unroll 4
      for (int k = 0; k < kKT; ++k) {
        float a[TM], bb[8];
#pragma unroll
        for (int i = 0; i < TM; ++i) a[i] = hs[(k0 + k) * C + ty * TM + i];
#pragma unroll
        for (int j = 0; j < 8; ++j) bb[j] = ws[k * 128 + tx * 8 + j];
#pragma unroll
        for (int i = 0; i < TM; ++i)
#pragma unroll
          for (int j = 0; j < 8; ++j) vacc[i][j] = fmaf(a[i], bb[j], vacc[i][j]);
      }
    }
  }

  // delta = V - Vhat for the thread's TM tokens x 8 dims
  const __nv_bfloat16* vrow = values + (unit * N + (size_t)c * C) * kEncD;
#pragma unroll
  for (int i = 0; i < TM; ++i) {
    const int t = ty * TM + i;
    float v[8], dl[8];
    load_bf16x8(vrow + (size_t)t * kEncD + tx * 8, v);
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      dl[j] = v[j] - vacc[i][j];
      ss = fmaf(dl[j], dl[j], ss);
    }
    if (!EMIT) {
#pragma unroll
      for (int o = 1; o < TX; o <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      if (tx == 0) norms[unit * N + (size_t)c * C + t] = sqrtf(ss);
    } else {
      const bool f = fl[t] != 0;   // uniform over the TX threads of the row
      if (!f) continue;
      int before = 0;
      for (int u = 0; u < t; ++u) before += fl[u];
      const size_t rec = (size_t)res_ptr[unit * (nC + 1) + c] + before;
      if (tx == 0) res_pos[rec] = (uint16_t)t;
      if (I8) {
        float m = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) m = fmaxf(m, fabsf(dl[j]));
        // the 16 threads of the row are 16 consecutive lanes of one warp
#pragma unroll
        for (int o = 1; o < TX; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0x0000ffffu << (threadIdx.x & 16), m, o));
        __half sh;
        uint2 codes;
        quantize8(dl, m, &sh, &codes, nullptr);
        *reinterpret_cast<uint2*>(static_cast<int8_t*>(res_val) + rec * kEncD + tx * 8) = codes;
        if (tx == 0) res_scale[rec] = sh;
      } else {
        *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(res_val) + rec * kEncD + tx * 8) = pack_bf16x8(dl);
      }
    }
  }
  (void)n_res;
}

// ----------------------------------------------------------------------- selection
// One CTA per unit; thread i owns tokens [i*TPT, (i+1)*TPT) so that a block scan in thread
// order is a scan in token order.  Radix select on the order key ~bits(norm) (norms are
// >= 0, so their bits order like the values): 8 bits a pass, it finds the n_res-th smallest
// key K and how many keys equal to K are still to take; those go to the lowest tokens.
constexpr int kSelThreads = 1024;

__device__ __forceinline__ int block_excl_scan(int v, int* wsum, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wsum[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int s = lane < (int)(blockDim.x >> 5) ? wsum[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    wsum[lane] = s;   // inclusive warp prefix
  }
  __syncthreads();
  total = wsum[(blockDim.x >> 5) - 1];
  const int excl = x - v + (warp > 0 ? wsum[warp - 1] : 0);
  __syncthreads();
  return excl;
}

__global__ void __launch_bounds__(kSelThreads)
enc_select_kernel(int N, int C, int n_res, const float* __restrict__ norms, uint8_t* __restrict__ flags,
                  int32_t* __restrict__ res_ptr) {
  __shared__ int hist[256];
  __shared__ int wsum[32];
  __shared__ int state[2];
  extern __shared__ int ccount[];   // [nC]
  const size_t unit = blockIdx.x;
  const int tid = threadIdx.x;
  const int nC = N / C;
  const int TPT = (N + kSelThreads - 1) / kSelThreads;
  const int t0 = tid * TPT, t1 = min(t0 + TPT, N);
  const float* nr = norms + unit * N;
  uint32_t prefix = 0;
  int kk = n_res;
  if (n_res > 0 && n_res < N) {
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int i = tid; i < 256; i += kSelThreads) hist[i] = 0;
      __syncthreads();
      for (int t = t0; t < t1; ++t) {
        const uint32_t k32 = ~__float_as_uint(nr[t]);
        if (shift == 24 || (k32 >> (shift + 8)) == (prefix >> (shift + 8))) atomicAdd(&hist[(k32 >> shift) & 255], 1);
      }
      __syncthreads();
      if (tid < 32) {   // one warp finds the bin holding the kk-th key
        int run = 0;
        for (int base = 0; base < 256; base += 32) {
          const int hv = hist[base + tid];
          int x = hv;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (tid >= o) x += y;
          }
          const int incl = run + x, excl = incl - hv;
          const unsigned hit = __ballot_sync(0xffffffffu, excl < kk && incl >= kk);
          if (hit) {
            const int w = __ffs(hit) - 1;
            const int ex = __shfl_sync(0xffffffffu, excl, w);
            if (tid == 0) {
              state[0] = base + w;
              state[1] = ex;
            }
            break;
          }
          run += __shfl_sync(0xffffffffu, x, 31);
        }
      }
      __syncthreads();
      prefix |= (uint32_t)state[0] << shift;
      kk -= state[1];
      __syncthreads();
    }
  }
  // flags: keys below the threshold, or equal to it and among the kk lowest such tokens
  int neq = 0;
  if (n_res > 0 && n_res < N)
    for (int t = t0; t < t1; ++t) neq += (~__float_as_uint(nr[t])) == prefix;
  int tot;
  int eqrank = block_excl_scan(neq, wsum, tot);
  for (int i = tid; i < nC; i += kSelThreads) ccount[i] = 0;
  __syncthreads();
  for (int t = t0; t < t1; ++t) {
    bool f;
    if (n_res >= N) {
      f = true;
    } else if (n_res <= 0) {
      f = false;
    } else {
      const uint32_t k32 = ~__float_as_uint(nr[t]);
      f = k32 < prefix || (k32 == prefix && eqrank++ < kk);
    }
    flags[unit * N + t] = f ? 1 : 0;
    if (f) atomicAdd(&ccount[t / C], 1);
  }
  __syncthreads();
  // CSR offsets of the unit's chunks: unit u's records start at u * n_res
  if (tid == 0) {
    int run = (int)(unit * (size_t)n_res);
    int32_t* rp = res_ptr + unit * (nC + 1);
    for (int c2 = 0; c2 < nC; ++c2) {
      rp[c2] = run;
      run += ccount[c2];
    }
    rp[nC] = run;
  }
}

// ------------------------------------------------------------- tensor-core residuals
// One persistent CTA per SM walks a contiguous range of tiles (unit, chunk), units ordered
// (layer, KV head, sequence) so that W1' and W2 are reloaded only when the (layer, KV head)
// changes.  Per tile, in order (every step waits for the previous one):
//   TMA: the chunk's stored coefficient tile (C rows x R, 128-byte swizzle, K-major)
//   MMA: D1_hh = (W1'_hh / 2) . A^T for hidden halves hh = 0, 1 (SS, M=128, N=C, K=R)
//   warps 0-3 / 4-7: H_hh = silu(2 D1_hh) = u + u tanh(u) as fp16, written to shared memory
//        MN-major (hidden rows, token-contiguous, 128-byte swizzle) -- half 0 over the A tile
//   MMA: D2 = W2 . H (SS, M=128 value dims, N=C, K=256; W2 in fp16, K-major)
//   warps: delta = V - D2 per (dim, token); norms (pass 1) or the flagged rows (pass 2)
// TMEM columns: D1 half 0 [0, C), half 1 [C, 2C), D2 [2C, 3C).
template <int R, int C>
struct EncTcLayout {
  static constexpr int KSLABS = R / 64;
  static constexpr int W1_HALF = KSLABS * 16384;          // 128 hidden rows x R, bf16
  static constexpr int W2_BYTES = 4 * 16384;              // 128 dims x 256 hidden, fp16
  static constexpr int H_HALF = (C / 64) * 16384;         // 128 hidden rows x C tokens, fp16
  static constexpr int A_BYTES = KSLABS * 16384;
  static constexpr int OFF_W1 = 0;
  static constexpr int OFF_W2 = OFF_W1 + 2 * W1_HALF;
  static constexpr int OFF_AH = OFF_W2 + W2_BYTES;        // the A tile, then H half 0
  static constexpr int OFF_H1 = OFF_AH + (A_BYTES > H_HALF ? A_BYTES : H_HALF);
  static constexpr int OFF_MISC = OFF_H1 + H_HALF;
  static constexpr int MISC_BYTES = 64 + 4 * C * 4 + 2 * C * 4;
  static constexpr int SMEM = OFF_MISC + MISC_BYTES + 1024;
  static_assert(SMEM <= 227 * 1024, "shared memory");
};

struct EncTcMisc {
  uint64_t bar_w, bar_in, bar_mma;
  uint32_t tmem_base;
  int abort_flag;
};

template <int R, int C, bool EMIT>
__global__ void __launch_bounds__(kEncThreads, 1)
enc_resid_tc_kernel(int B, int L, int G, int Hkv, int N, const __grid_constant__ CUtensorMap tmW1,
                    const __grid_constant__ CUtensorMap tmW2, const __grid_constant__ CUtensorMap tmA,
                    const __nv_bfloat16* __restrict__ values, float* __restrict__ norms,
                    const uint8_t* __restrict__ flags, const int32_t* __restrict__ res_ptr,
                    uint16_t* __restrict__ res_pos, __nv_bfloat16* __restrict__ res_val, uint32_t* err) {
  using namespace tc;
  using Lay = EncTcLayout<R, C>;
  extern __shared__ unsigned char enc_smem_dyn[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(enc_smem_dyn) + 1023) & ~uintptr_t(1023));
  EncTcMisc* misc = reinterpret_cast<EncTcMisc*>(smem + Lay::OFF_MISC);
  float* part = reinterpret_cast<float*>(smem + Lay::OFF_MISC + 64);   // [4][C]
  int* fl = reinterpret_cast<int*>(part + 4 * C);                       // [C]
  int* pfx = fl + C;                                                    // [C]
  volatile int* abort_flag = &misc->abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nC = N / C, NG = L / G;
  const long long total = (long long)B * L * Hkv * nC;
  const long long x0 = total * blockIdx.x / gridDim.x, x1 = total * (blockIdx.x + 1) / gridDim.x;

  if (tid == 0) {
    mbar_init(&misc->bar_w, 1);
    mbar_init(&misc->bar_in, 1);
    mbar_init(&misc->bar_mma, 1);
    misc->abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == 0) {
    tmem_alloc(&misc->tmem_base, 512);
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc->tmem_base;
  const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
  const uint64_t dW1 = smem_desc(smem_u32(smem + Lay::OFF_W1), 16, 1024, 2);
  const uint64_t dW2 = smem_desc(smem_u32(smem + Lay::OFF_W2), 16, 1024, 2);
  const uint64_t dA = smem_desc(smem_u32(smem + Lay::OFF_AH), 16, 1024, 2);
  const uint64_t dH0 = smem_desc(smem_u32(smem + Lay::OFF_AH), 16384, 1024, 2);   // MN-major
  const uint64_t dH1 = smem_desc(smem_u32(smem + Lay::OFF_H1), 16384, 1024, 2);
  constexpr uint32_t IDESC_1 = idesc_f16(128, C, 1, 1);         // W1' (bf16) x A (bf16)
  constexpr uint32_t IDESC_2 = idesc_f16(128, C, 0, 0, 0, 1);   // W2 (f16) x H (f16, MN-major)
  uint32_t ph_w = 0, ph_in = 0, ph_mma = 0;
  int cur_seg = -1;
  bool ok = true;
  const int hh = warp >> 2;                 // epilogue 1: hidden half; epilogue 2: token half
  const int row = 32 * (warp & 3) + lane;   // TMEM lane: hidden unit in the half / value dim

  for (long long x = x0; ok && x < x1; ++x) {
    const int u = (int)(x / nC), c = (int)(x % nC);
    const int b = u % B, seg = u / B, hkv = seg % Hkv, l = seg / Hkv, grp = l / G;
    const size_t unit = ((size_t)b * L + l) * Hkv + hkv;
    if (seg != cur_seg) {   // W1' halves and W2 of this (layer, KV head)
      if (tid == 0) {
        mbar_expect_tx(&misc->bar_w, (uint32_t)(2 * Lay::W1_HALF + Lay::W2_BYTES));
        for (int h2 = 0; h2 < 2; ++h2)
          for (int ks = 0; ks < Lay::KSLABS; ++ks)
            tma_load_2d(smem + Lay::OFF_W1 + h2 * Lay::W1_HALF + ks * 16384, &tmW1, &misc->bar_w, ks * 64,
                        seg * 256 + h2 * 128);
        for (int j = 0; j < 4; ++j)
          tma_load_2d(smem + Lay::OFF_W2 + j * 16384, &tmW2, &misc->bar_w, j * 64, seg * 128);
      }
      ok = mbar_wait(&misc->bar_w, ph_w, abort_flag, err, ERR_TIMEOUT);
      ph_w ^= 1;
      cur_seg = seg;
      if (!__syncthreads_and(ok)) break;
    }
    const long long arow = (((long long)b * NG + grp) * Hkv + hkv) * N + (long long)c * C;
    if (tid == 0) {
      mbar_expect_tx(&misc->bar_in, (uint32_t)(Lay::KSLABS * C * 128));
      for (int ks = 0; ks < Lay::KSLABS; ++ks)
        tma_load_2d(smem + Lay::OFF_AH + ks * 16384, &tmA, &misc->bar_in, ks * 64, (int)arow);
    }
    if (EMIT)
      for (int t = tid; t < C; t += kEncThreads) fl[t] = flags[unit * N + (size_t)c * C + t];
    // this thread's values for the residual epilogue (dim `row`, tokens hh*C/2 .. +C/2),
    // requested now so that they arrive during the MMAs
    uint32_t vv[C / 4];
    {
      const unsigned short* vrow = reinterpret_cast<const unsigned short*>(values) +
                                   (unit * N + (size_t)c * C + hh * (C / 2)) * kEncD + row;
#pragma unroll
      for (int j = 0; j < C / 4; ++j)
        vv[j] = (uint32_t)__ldg(vrow + (size_t)(2 * j) * kEncD) | ((uint32_t)__ldg(vrow + (size_t)(2 * j + 1) * kEncD) << 16);
    }
    ok = mbar_wait(&misc->bar_in, ph_in, abort_flag, err, ERR_TIMEOUT);
    ph_in ^= 1;
    if (!__syncthreads_and(ok)) break;
    // D1 of both hidden halves
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2)
#pragma unroll
        for (int kk = 0; kk < R / 16; ++kk) {
          const uint64_t ko = (uint64_t)((kk >> 2) * 1024 + (kk & 3) * 2);
          mma_ss(tmem + h2 * C, dW1 + (uint64_t)((h2 * Lay::W1_HALF) >> 4) + ko, dA + ko, IDESC_1, kk > 0 ? 1u : 0u);
        }
      mma_commit(&misc->bar_mma);
    }
    ok = mbar_wait(&misc->bar_mma, ph_mma, abort_flag, err, ERR_TIMEOUT);
    ph_mma ^= 1;
    if (!__syncthreads_and(ok)) break;
    tc_fence_after();
    // silu -> H_hh (fp16) in shared memory, MN-major: hidden row `row`, 8 tokens per 16 bytes
    {
      unsigned char* hrow = smem + (hh == 0 ? Lay::OFF_AH : Lay::OFF_H1) + (row >> 3) * 1024 + (row & 7) * 128;
#pragma unroll
      for (int q = 0; q < C / 32; ++q) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_off + hh * C + q * 32, v);
        tmem_wait_ld();
        uint32_t h[16];
#pragma unroll
        for (int j = 0; j < 16; ++j)
          h[j] = silu_half2_of_halfx(pack_f16x2(__uint_as_float(v[2 * j]), __uint_as_float(v[2 * j + 1])));
        unsigned char* blk = hrow + (q >> 1) * 16384;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int c16 = (q & 1) * 4 + k;
          *reinterpret_cast<uint4*>(blk + ((c16 ^ (row & 7)) << 4)) = make_uint4(h[4 * k], h[4 * k + 1], h[4 * k + 2], h[4 * k + 3]);
        }
      }
    }
    tc_fence_before();
    fence_proxy_async_smem();
    __syncthreads();
    // D2 = W2 . H over both hidden halves
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2)
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const int slab = h2 * 2 + (kk >> 2);
          mma_ss(tmem + 2 * C, dW2 + (uint64_t)((slab * 16384 + (kk & 3) * 32) >> 4),
                 (h2 == 0 ? dH0 : dH1) + (uint64_t)((kk * 2048) >> 4), IDESC_2, (h2 | kk) ? 1u : 0u);
        }
      mma_commit(&misc->bar_mma);
    }
    if (EMIT && tid < C) {   // rank of each token among the chunk's flagged tokens
      int s = 0;
      for (int t = 0; t < tid; ++t) s += fl[t];
      pfx[tid] = s;
    }
    ok = mbar_wait(&misc->bar_mma, ph_mma, abort_flag, err, ERR_TIMEOUT);
    ph_mma ^= 1;
    if (!__syncthreads_and(ok)) break;   // (also publishes pfx)
    tc_fence_after();
    // delta = V - Vhat for dim `row`, tokens hh*C/2 .. +C/2
    const size_t rbase = EMIT ? (size_t)res_ptr[unit * (nC + 1) + c] : 0;
#pragma unroll
    for (int q = 0; q < C / 64; ++q) {
      uint32_t v[32];
      tmem_ld32(tmem + lane_off + 2 * C + hh * (C / 2) + q * 32, v);
      tmem_wait_ld();
      float ss[32];   // pass 1: this lane's d^2 for the 32 tokens of the slice
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int t = hh * (C / 2) + q * 32 + j;
        const uint32_t w = vv[(q * 32 + j) >> 1];
        const float vt = __uint_as_float(((j & 1) ? (w >> 16) : (w & 0xffffu)) << 16);
        const float d = vt - __uint_as_float(v[j]);
        if (!EMIT) {
          ss[j] = d * d;
        } else if (fl[t]) {
          const size_t rec = rbase + pfx[t];
          res_val[rec * kEncD + row] = __float2bfloat16_rn(d);
          if (row == 0) res_pos[rec] = (uint16_t)t;
        }
      }
      if (!EMIT) {
        // sums over the warp's 32 dims for 32 tokens with 31 shuffles (a transposing
        // butterfly: at distance o a lane keeps the half of its partial sums whose token
        // index has bit o equal to its own, adds the partner's, and passes the other half),
        // after which lane L holds token L's sum
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
          const bool up = (lane & o) != 0;
#pragma unroll
          for (int i = 0; i < o; ++i) {
            const float keep = up ? ss[i + o] : ss[i];
            const float give = up ? ss[i] : ss[i + o];
            ss[i] = keep + __shfl_xor_sync(0xffffffffu, give, o);
          }
        }
        part[(warp & 3) * C + hh * (C / 2) + q * 32 + lane] = ss[0];
      }
    }
    tc_fence_before();
    __syncthreads();
    if (!EMIT)
      for (int t = tid; t < C; t += kEncThreads)
        norms[unit * N + (size_t)c * C + t] = sqrtf(part[t] + part[C + t] + part[2 * C + t] + part[3 * C + t]);
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------- tensor-core residuals, C = 128, tokens as M
// The same pass with the chunk's 128 tokens as the MMAs' M dimension, so that every
// per-token step of the epilogue (the token's values row against its rebuilt row, the norm
// of the difference, a bf16 record) is local to one thread (an int8 record's scale and codes
// are computed by the token's warp together, four dims per lane):
//   D1^T = A . (W1'/2)^T (SS, M = 128 tokens, N = 128 per hidden half, K = R)
//   H^T  = silu(2 D1^T) as fp16 pairs, written over the first 128 of the tile's TMEM columns
//          (thread = token: its 256 hidden units)
//   D2^T = H^T . W2^T    (TS: A = H from TMEM, B = W2 in fp16, K-major; M = 128 tokens,
//          N = 128 value dims, K = 256), into the tile's columns 128..255
// Two tiles in flight: tile i of the CTA's range uses TMEM columns [256 (i%2), +256) and
// coefficient stage i%2; warps 0-3 take the even tiles, 4-7 the odd ones; warp 8 issues the
// copies and the MMAs, the next tile's pre-activations before this tile's second GEMM.
constexpr int kEnc2Threads = 288;

template <int R, bool I8 = false>
struct EncTc2Layout {
  static constexpr int KSLABS = R / 64;
  static constexpr int W1_HALF = KSLABS * 16384;          // 128 hidden rows x R, 16-bit
  static constexpr int W2_BYTES = 4 * 16384;              // 128 dims x 256 hidden, fp16
  static constexpr int A_BYTES = KSLABS * 16384;          // 128 tokens x R, 16-bit
  static constexpr int SA_SLOT = 128 * R + 128 * 2;       // int8 store: the int8 tile + row scales
  static constexpr int OFF_W1 = 0;
  static constexpr int OFF_W2 = OFF_W1 + 2 * W1_HALF;
  static constexpr int OFF_A = OFF_W2 + W2_BYTES;         // two stages
  static constexpr int OFF_SA = OFF_A + 2 * A_BYTES;      // int8 store: two staging slots
  static constexpr int OFF_MISC = OFF_SA + (I8 ? 2 * SA_SLOT : 0);
  static constexpr int SMEM = OFF_MISC + 256 + 1024;
  static_assert(SMEM <= 227 * 1024, "shared memory");
};

struct EncTc2Misc {
  uint64_t w_full, drain, a_full[2], a_empty[2], d1_full[2], h_ready[2], d2_full[2], slot_free[2], a_conv[2];
  uint32_t tmem_base;
  int abort_flag;
};

// I8 (int8 store): the stored int8 rows and their scales arrive by bulk copies into a staging
// slot, and each thread of the tile's group writes its own token's row sigma_t a_t as fp16
// (int8 times the fp16 scale is exact in fp32, rounded once) into the coefficient stage the
// MMAs read; W1'/2 is then fp16 too, and the residual record is the int8 row with its scale.
template <int R, bool EMIT, bool I8 = false>
__global__ void __launch_bounds__(kEnc2Threads, 1)
enc_resid_tc2_kernel(int B, int L, int G, int Hkv, int N, const __grid_constant__ CUtensorMap tmW1,
                     const __grid_constant__ CUtensorMap tmW2, const __grid_constant__ CUtensorMap tmA,
                     const void* __restrict__ coeff, const __half* __restrict__ coeff_scale,
                     const __nv_bfloat16* __restrict__ values, float* __restrict__ norms,
                     const uint8_t* __restrict__ flags, const int32_t* __restrict__ res_ptr,
                     uint16_t* __restrict__ res_pos, void* __restrict__ res_val, __half* __restrict__ res_scale,
                     uint32_t* err) {
  using namespace tc;
  constexpr int C = 128;
  using Lay = EncTc2Layout<R, I8>;
  extern __shared__ unsigned char enc2_smem_dyn[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(enc2_smem_dyn) + 1023) & ~uintptr_t(1023));
  EncTc2Misc* misc = reinterpret_cast<EncTc2Misc*>(smem + Lay::OFF_MISC);
  volatile int* abort_flag = &misc->abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nC = N / C, NG = L / G;
  const long long total = (long long)B * L * Hkv * nC;
  const long long x0 = total * blockIdx.x / gridDim.x, x1 = total * (blockIdx.x + 1) / gridDim.x;
  const long long n = x1 - x0;

  if (tid == 0) {
    mbar_init(&misc->w_full, 1);
    mbar_init(&misc->drain, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&misc->a_full[s], 1);
      mbar_init(&misc->a_empty[s], 1);
      mbar_init(&misc->d1_full[s], 1);
      mbar_init(&misc->h_ready[s], 4);     // the 4 warps of the tile's group
      mbar_init(&misc->d2_full[s], 1);
      mbar_init(&misc->slot_free[s], 4);
      mbar_init(&misc->a_conv[s], 4);      // the group's converted rows (int8 store)
    }
    misc->abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == 8) {
    tmem_alloc(&misc->tmem_base, 512);
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc->tmem_base;

  if (warp == 8) {
    // ============================================================ copies and MMAs
    const bool leader = elect_one();
    const uint64_t dW1 = smem_desc(smem_u32(smem + Lay::OFF_W1), 16, 1024, 2);
    const uint64_t dW2 = smem_desc(smem_u32(smem + Lay::OFF_W2), 16, 1024, 2);
    const uint64_t dA0 = smem_desc(smem_u32(smem + Lay::OFF_A), 16, 1024, 2);
    // A x W1'/2, both K-major: bf16, or fp16 for the int8 store
    constexpr uint32_t IDESC_1 = I8 ? idesc_f16(128, 128, 0, 0) : idesc_f16(128, 128, 1, 1);
    constexpr uint32_t IDESC_2 = idesc_f16(128, 128, 0, 0);   // H (TMEM, fp16) x W2 (fp16, K-major)
    auto wait_all = [&](uint64_t* bar, uint32_t par) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, par, abort_flag, err, ERR_TIMEOUT));
    };
    auto seg_of = [&](long long i) { return (int)((x0 + i) / nC / B); };
    auto issue_a = [&](long long i) {   // tile i's coefficient tile into stage (or staging slot) i % 2
      const long long x = x0 + i;
      const int u = (int)(x / nC), c = (int)(x % nC);
      const int b = u % B, seg = u / B, hkv = seg % Hkv, l = seg / Hkv, grp = l / G;
      const long long arow = (((long long)b * NG + grp) * Hkv + hkv) * N + (long long)c * C;
      if (leader) {
        if (I8) {
          unsigned char* dst = smem + Lay::OFF_SA + (i & 1) * Lay::SA_SLOT;
          mbar_expect_tx(&misc->a_full[i & 1], (uint32_t)Lay::SA_SLOT);
          bulk_load(dst, static_cast<const int8_t*>(coeff) + arow * R, (uint32_t)(C * R), &misc->a_full[i & 1]);
          bulk_load(dst + C * R, coeff_scale + arow, (uint32_t)(C * 2), &misc->a_full[i & 1]);
        } else {
          mbar_expect_tx(&misc->a_full[i & 1], (uint32_t)Lay::A_BYTES);
          for (int ks = 0; ks < Lay::KSLABS; ++ks)
            tma_load_2d(smem + Lay::OFF_A + (i & 1) * Lay::A_BYTES + ks * 16384, &tmA, &misc->a_full[i & 1],
                        ks * 64, (int)arow);
        }
      }
      __syncwarp();
    };
    uint32_t ph_w = 0, ph_drain = 0;
    long long a_waited = 0, a_issued = 0;   // coefficient copies consumed / issued
    bool ok = true, w_pending = false;
    auto load_w = [&](int seg) -> bool {   // W1' halves and W2 of this (layer, KV head)
      w_pending = true;
      if (leader) {
        mbar_expect_tx(&misc->w_full, (uint32_t)(2 * Lay::W1_HALF + Lay::W2_BYTES));
        for (int h2 = 0; h2 < 2; ++h2)
          for (int ks = 0; ks < Lay::KSLABS; ++ks)
            tma_load_2d(smem + Lay::OFF_W1 + h2 * Lay::W1_HALF + ks * 16384, &tmW1, &misc->w_full, ks * 64,
                        seg * 256 + h2 * 128);
        for (int j = 0; j < 4; ++j) tma_load_2d(smem + Lay::OFF_W2 + j * 16384, &tmW2, &misc->w_full, j * 64, seg * 128);
      }
      __syncwarp();
      if (!wait_all(&misc->w_full, ph_w)) return false;
      ph_w ^= 1;
      w_pending = false;
      return true;
    };
    auto issue_d1 = [&](long long i) -> bool {
      const int s = (int)(i & 1);
      // the tile in the stage: by TMA, or (int8 store) converted by its group from the staging
      // slot, which the group waited for (so the copy has landed either way)
      if (!wait_all(I8 ? &misc->a_conv[s] : &misc->a_full[s], (uint32_t)((i >> 1) & 1))) return false;
      a_waited = i + 1;
      if (i >= 2 && !wait_all(&misc->slot_free[s], (uint32_t)(((i >> 1) - 1) & 1))) return false;
      if (leader) {
        tc_fence_after();
        const uint64_t dA = dA0 + (uint64_t)((s * Lay::A_BYTES) >> 4);
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2)
#pragma unroll
          for (int kk = 0; kk < R / 16; ++kk) {
            const uint64_t ko = (uint64_t)((kk >> 2) * 1024 + (kk & 3) * 2);
            mma_ss(tmem + 256 * s + h2 * 128, dA + ko, dW1 + (uint64_t)((h2 * Lay::W1_HALF) >> 4) + ko, IDESC_1,
                   kk > 0 ? 1u : 0u);
          }
        mma_commit(&misc->d1_full[s]);
        mma_commit(&misc->a_empty[s]);
      }
      __syncwarp();
      return true;
    };
    auto issue_d2 = [&](long long i) -> bool {
      const int s = (int)(i & 1);
      if (!wait_all(&misc->h_ready[s], (uint32_t)((i >> 1) & 1))) return false;
      if (leader) {
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 16; ++kk)
          mma_ts(tmem + 256 * s + 128, tmem + 256 * s + kk * 8,
                 dW2 + (uint64_t)(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4), IDESC_2, kk > 0 ? 1u : 0u);
        mma_commit(&misc->d2_full[s]);
      }
      __syncwarp();
      return true;
    };
    auto drain_mmas = [&](volatile int* flag) -> bool {   // every MMA issued so far is complete
      if (leader) mma_commit(&misc->drain);
      __syncwarp();
      const bool r = __all_sync(0xffffffffu, mbar_wait(&misc->drain, ph_drain, flag, err, ERR_TIMEOUT));
      ph_drain ^= 1;
      return r;
    };
    if (n > 0) {
      issue_a(0);
      a_issued = 1;
      if (n > 1) {
        issue_a(1);
        a_issued = 2;
      }
      int cur_seg = seg_of(0);
      ok = load_w(cur_seg) && issue_d1(0);
      for (long long i = 0; ok && i < n; ++i) {
        const bool has_next = i + 1 < n;
        const bool same = has_next && seg_of(i + 1) == cur_seg;
        if (same && !(ok = issue_d1(i + 1))) break;   // the next tile's pre-activations first
        if (!(ok = issue_d2(i))) break;
        if (has_next && !same) {   // a new (layer, KV head): W1', W2 reloaded once no MMA reads them
          if (!(ok = drain_mmas(abort_flag))) break;
          cur_seg = seg_of(i + 1);
          if (!(ok = load_w(cur_seg) && issue_d1(i + 1))) break;
        }
        // tile i's stage is free once its pre-activations are done: tile i + 2 goes there
        if (i + 2 < n) {
          if (!(ok = wait_all(&misc->a_empty[i & 1], (uint32_t)((i >> 1) & 1)))) break;
          issue_a(i + 2);
          a_issued = i + 3;
        }
      }
      // before the CTA's TMEM and shared memory go: every MMA and copy it started is done
      volatile int never = 0;
      drain_mmas(&never);
      if (!ok && leader) {
        for (long long i = a_waited; i < a_issued; ++i)
          mbar_wait(&misc->a_full[i & 1], (uint32_t)((i >> 1) & 1), &never, err, ERR_TIMEOUT);
        if (w_pending) mbar_wait(&misc->w_full, ph_w, &never, err, ERR_TIMEOUT);   // a W1' / W2 copy in flight
      }
    }
  } else {
    // ============================================================ silu and epilogue
    const int grp_t = warp >> 2;                       // tiles i with i % 2 == grp_t
    const int wq = warp & 3;
    const int t = 32 * wq + lane;                      // this thread's token (TMEM lane)
    const uint32_t lane_off = (uint32_t)(32 * wq) << 16;
    const unsigned lt_mask = (1u << lane) - 1u;
    for (long long i = grp_t; i < n; i += 2) {
      const long long x = x0 + i;
      const int s = (int)(i & 1);
      const uint32_t par = (uint32_t)((i >> 1) & 1);
      const int u = (int)(x / nC), c = (int)(x % nC);
      const int b = u % B, seg = u / B, hkv = seg % Hkv, l = seg / Hkv;
      const size_t unit = ((size_t)b * L + l) * Hkv + hkv;
      const size_t tok = unit * N + (size_t)c * C;   // the chunk's first token
      int flagged = 0, rank = 0, rank0 = 0;   // rank0: flagged tokens of the earlier warps
      unsigned fb = 0;                        // this warp's flagged lanes
      size_t rbase = 0;
      if (EMIT) {   // the token's rank among the chunk's flagged tokens: one ballot per warp
#pragma unroll
        for (int w4 = 0; w4 < 4; ++w4) {
          const unsigned bw = __ballot_sync(0xffffffffu, flags[tok + 32 * w4 + lane] != 0);
          if (w4 < wq) rank0 += __popc(bw);
          if (w4 == wq) fb = bw;
        }
        flagged = (fb >> lane) & 1u;
        rank = rank0 + __popc(fb & lt_mask);
        rbase = (size_t)res_ptr[unit * (nC + 1) + c];
      }
      // the token's values row for the epilogue (pass 2: flagged tokens only), requested now;
      // for an int8 record copied into shared memory once the silu is done (below), so that
      // it does not sit in registers through the conversion and the silu
      uint4 vrow[kEncD / 8];
      const uint4* vp = reinterpret_cast<const uint4*>(values + (tok + t) * kEncD);
      if (!(EMIT && I8)) {
#pragma unroll
        for (int j = 0; j < kEncD / 8; ++j) vrow[j] = (!EMIT || flagged) ? __ldg(vp + j) : make_uint4(0, 0, 0, 0);
      }
      if (I8) {   // this token's stored row, sigma_t a_t as fp16, into the coefficient stage
        // pass 2 stages the flagged tokens' rows in this stage (below), and a warp's slots
        // there overlap other warps' coefficient rows (r = 128): the group's previous tile must
        // be done by all four warps (their slot_free arrivals) before any of them overwrites it
        if (EMIT && i >= 2 &&
            !__all_sync(0xffffffffu, mbar_wait(&misc->slot_free[s], par ^ 1u, abort_flag, err, ERR_TIMEOUT)))
          break;
        if (!__all_sync(0xffffffffu, mbar_wait(&misc->a_full[s], par, abort_flag, err, ERR_TIMEOUT))) break;
        const unsigned char* src = smem + Lay::OFF_SA + s * Lay::SA_SLOT;
        const float sg = __half2float(reinterpret_cast<const __half*>(src + C * R)[t]);
        unsigned char* arow_s = smem + Lay::OFF_A + s * Lay::A_BYTES + t * 128;
#pragma unroll
        for (int j = 0; j < R / 8; ++j) {   // 8 values = one 16-byte chunk of the swizzled row
          const uint2 q = *reinterpret_cast<const uint2*>(src + t * R + 8 * j);
          const uint32_t qw[2] = {q.x, q.y};
          uint32_t o[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float x0f = (float)(int8_t)((qw[k >> 1] >> (16 * (k & 1))) & 0xffu) * sg;
            const float x1f = (float)(int8_t)((qw[k >> 1] >> (16 * (k & 1) + 8)) & 0xffu) * sg;
            const __half2 h2 = __floats2half2_rn(x0f, x1f);
            o[k] = *reinterpret_cast<const uint32_t*>(&h2);
          }
          const int ks = j >> 3, jj = j & 7;
          *reinterpret_cast<uint4*>(arow_s + ks * 16384 + ((jj ^ (t & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&misc->a_conv[s]);
      }
      if (!__all_sync(0xffffffffu, mbar_wait(&misc->d1_full[s], par, abort_flag, err, ERR_TIMEOUT))) break;
      tc_fence_after();
      // H = silu(2 D1) for this token's 256 hidden units, as fp16 pairs over columns 0..127
      // (64 columns per TMEM round trip; the writes of a pair of chunks land on columns both
      // chunks have already been read from)
#pragma unroll
      for (int q = 0; q < 8; q += 2) {
        uint32_t v[32], v2[32];
        tmem_ld32(tmem + lane_off + 256 * s + 32 * q, v);
        tmem_ld32(tmem + lane_off + 256 * s + 32 * q + 32, v2);
        tmem_wait_ld();
        uint32_t h[16];
#pragma unroll
        for (int j = 0; j < 16; ++j)
          h[j] = silu_half2_of_halfx(pack_f16x2(__uint_as_float(v[2 * j]), __uint_as_float(v[2 * j + 1])));
        tmem_st16(tmem + lane_off + 256 * s + 16 * q, h);
#pragma unroll
        for (int j = 0; j < 16; ++j)
          h[j] = silu_half2_of_halfx(pack_f16x2(__uint_as_float(v2[2 * j]), __uint_as_float(v2[2 * j + 1])));
        tmem_st16(tmem + lane_off + 256 * s + 16 * q + 16, h);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&misc->h_ready[s]);
      // int8 record (pass 2): each warp quantises its flagged tokens' rows together, four
      // dims per lane, instead of each row by its own lane.  The warp's quarter of this tile's
      // coefficient stage (free: the pre-activations are done, and the group's next conversion
      // waits for this tile's slot_free) holds kNSlot row slots of 512 bytes; the flagged token
      // of warp rank m < kNSlot copies its values row (bf16) into the upper half of slot m now,
      // while the second GEMM runs, 16-byte piece j at (16 + j) ^ (m % 8).
      constexpr int kQB = Lay::A_BYTES / 4, kNSlot = kQB / 512;
      unsigned char* wbase = smem + Lay::OFF_A + s * Lay::A_BYTES + wq * kQB;
      const int wrank = __popc(fb & lt_mask), kw = __popc(fb);
      auto stage_v = [&](int m) {
        unsigned char* slot = wbase + m * 512;
#pragma unroll
        for (int j = 0; j < kEncD / 8; ++j)
          asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(slot + (((16 + j) ^ (m & 7)) << 4))),
                       "l"(vp + j)
                       : "memory");
        asm volatile("cp.async.commit_group;" ::: "memory");
      };
      if (EMIT && I8 && flagged && wrank < kNSlot) stage_v(wrank);
      if (!__all_sync(0xffffffffu, mbar_wait(&misc->d2_full[s], par, abort_flag, err, ERR_TIMEOUT))) {
        if (EMIT && I8) asm volatile("cp.async.wait_all;" ::: "memory");   // no copy outlives the CTA
        break;
      }
      tc_fence_after();
      // delta = V - Vhat for this token's 128 dims: its norm (pass 1) or its record (pass 2)
      float ss = 0.f;
      if constexpr (EMIT && I8) {
        // per batch of up to kNSlot flagged tokens: each writes its delta row (fp32) into its
        // slot, 16-byte piece p (dims 4p .. 4p + 3) at p ^ (m % 8) -- over the values row as it
        // is consumed (dims 32q .. 32q + 31 land on pieces 8q .. 8q + 7, which hold values of
        // dims below 32q only); then the warp takes the slots one by one: lane L the dims
        // 4L .. 4L + 3, the row's largest |delta| by a butterfly, its fp16 scale s, the codes
        // round-half-even of delta / s (code8_scaled), 128 bytes stored at once
        for (int b0 = 0; b0 < kw; b0 += kNSlot) {
          const bool mine = flagged && wrank >= b0 && wrank < b0 + kNSlot;
          const int m = wrank - b0;
          if (b0 > 0 && mine) stage_v(m);   // later batches (more than kNSlot flagged lanes)
          asm volatile("cp.async.wait_all;" ::: "memory");
          unsigned char* slot = wbase + (mine ? m : 0) * 512;
#pragma unroll 1
          for (int q = 0; q < kEncD / 32; ++q) {
            uint32_t vh[32];   // (warp-wide load; only this batch's lanes use it)
            tmem_ld32(tmem + lane_off + 256 * s + 128 + 32 * q, vh);
            tmem_wait_ld();
            if (!mine) continue;
            uint4 w4[4];   // values dims 32q .. 32q + 31, read before any delta of them is written
#pragma unroll
            for (int k8 = 0; k8 < 4; ++k8)
              w4[k8] = *reinterpret_cast<const uint4*>(slot + (((16 + 4 * q + k8) ^ (m & 7)) << 4));
#pragma unroll
            for (int k8 = 0; k8 < 4; ++k8) {
              const uint32_t ww[4] = {w4[k8].x, w4[k8].y, w4[k8].z, w4[k8].w};
              float x8[8];
#pragma unroll
              for (int h = 0; h < 4; ++h) {
                x8[2 * h] = __uint_as_float(ww[h] << 16) - __uint_as_float(vh[8 * k8 + 2 * h]);
                x8[2 * h + 1] = __uint_as_float(ww[h] & 0xffff0000u) - __uint_as_float(vh[8 * k8 + 2 * h + 1]);
              }
              const int p0 = 8 * q + 2 * k8;   // pieces p0, p0 + 1
              *reinterpret_cast<float4*>(slot + ((p0 ^ (m & 7)) << 4)) = make_float4(x8[0], x8[1], x8[2], x8[3]);
              *reinterpret_cast<float4*>(slot + (((p0 + 1) ^ (m & 7)) << 4)) =
                  make_float4(x8[4], x8[5], x8[6], x8[7]);
            }
          }
          __syncwarp();   // the batch's delta rows are visible to the whole warp
          const int nb = min(kNSlot, kw - b0);
#pragma unroll 1
          for (int mm = 0; mm < nb; ++mm) {
            const float4 xv = *reinterpret_cast<const float4*>(wbase + mm * 512 + ((lane ^ (mm & 7)) << 4));
            const float x4[4] = {xv.x, xv.y, xv.z, xv.w};
            float amax = fmaxf(fmaxf(fabsf(x4[0]), fabsf(x4[1])), fmaxf(fabsf(x4[2]), fabsf(x4[3])));
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
            const __half sh = __float2half_rn(amax / 127.f);
            const float sc = __half2float(sh), rc = sc > 0.f ? 1.f / sc : 0.f;
            uint32_t code = 0u;
#pragma unroll
            for (int k = 0; k < 4; ++k) code |= code8_scaled(x4[k], sc, rc) << (8 * k);
            const size_t rec = rbase + (size_t)(rank0 + b0 + mm);
            *reinterpret_cast<uint32_t*>(static_cast<int8_t*>(res_val) + rec * kEncD + 4 * lane) = code;
            if (lane == 0) res_scale[rec] = sh;
          }
          __syncwarp();   // every slot read before the next batch overwrites it
        }
      } else {
        uint32_t vd[kEncD];   // the token's rebuilt row, all of it in one TMEM round trip
#pragma unroll
        for (int q = 0; q < kEncD / 32; ++q)
          tmem_ld32(tmem + lane_off + 256 * s + 128 + 32 * q, *reinterpret_cast<uint32_t(*)[32]>(vd + 32 * q));
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < kEncD / 32; ++q) {
          const uint32_t* v = vd + 32 * q;
          uint32_t o[16];
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            const uint4 w4 = vrow[(32 * q + j) >> 3];
            const uint32_t w = ((j >> 1) & 3) == 0 ? w4.x : ((j >> 1) & 3) == 1 ? w4.y : ((j >> 1) & 3) == 2 ? w4.z : w4.w;
            const float d0 = __uint_as_float(w << 16) - __uint_as_float(v[j]);
            const float d1 = __uint_as_float(w & 0xffff0000u) - __uint_as_float(v[j + 1]);
            if (!EMIT) {
              ss = fmaf(d0, d0, ss);
              ss = fmaf(d1, d1, ss);
            } else {
              const __nv_bfloat162 p = __floats2bfloat162_rn(d0, d1);
              o[j >> 1] = *reinterpret_cast<const uint32_t*>(&p);
            }
          }
          if (EMIT && flagged) {
            uint4* dst =
                reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(res_val) + (rbase + rank) * kEncD + 32 * q);
#pragma unroll
            for (int k = 0; k < 4; ++k) dst[k] = make_uint4(o[4 * k], o[4 * k + 1], o[4 * k + 2], o[4 * k + 3]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&misc->slot_free[s]);
      if (!EMIT) norms[tok + t] = sqrtf(ss);
      if (EMIT && flagged) res_pos[rbase + rank] = (uint16_t)t;
    }
  }
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ----------------------------------------------------------- tensor-core coefficients
// Per (b, group, KV head, chunk) tile of 128 tokens: D = sum_{l in group} K_l . B_l^T (SS
// MMAs, M = 128 tokens, N = R, K = d in steps of 16), the key and basis slabs of layer l+1
// loaded by TMA while the MMAs of layer l run (two buffers).  Epilogue: thread = token row
// (TMEM lane), so an int8 row scale is thread-local; the chunk summary sums the stored
// rows through shared memory.  Persistent, one tile in flight.
template <int R>
struct EncCoeffLayout {
  static constexpr int BUF = 2 * 16384 + 2 * R * 128;   // key slabs (128 rows) + basis slabs (R rows)
  static constexpr int OFF_BUF = 0;
  static constexpr int OFF_SUM = 2 * BUF;                // [128][R] fp32 stored rows
  static constexpr int OFF_MISC = OFF_SUM + 128 * R * 4;
  static constexpr int SMEM = OFF_MISC + 64 + 1024;
  static_assert(SMEM <= 227 * 1024, "shared memory");
};

struct EncCoeffMisc {
  uint64_t bar_in[2], bar_mma[2];
  uint32_t tmem_base;
  int abort_flag;
};

template <int R, bool I8>
__global__ void __launch_bounds__(128, 1)
enc_coeff_tc_kernel(int B, int L, int G, int Hkv, int N, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmB, void* __restrict__ coeff,
                    __half* __restrict__ coeff_scale, __nv_bfloat16* __restrict__ summary, uint32_t* err) {
  using namespace tc;
  using Lay = EncCoeffLayout<R>;
  constexpr int C = 128;
  extern __shared__ unsigned char enc_smem_dyn[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(enc_smem_dyn) + 1023) & ~uintptr_t(1023));
  EncCoeffMisc* misc = reinterpret_cast<EncCoeffMisc*>(smem + Lay::OFF_MISC);
  float* rows = reinterpret_cast<float*>(smem + Lay::OFF_SUM);
  volatile int* abort_flag = &misc->abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int nC = N / C, NG = L / G;
  const long long total = (long long)B * NG * Hkv * nC;
  const long long x0 = total * blockIdx.x / gridDim.x, x1 = total * (blockIdx.x + 1) / gridDim.x;
  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&misc->bar_in[i], 1);
      mbar_init(&misc->bar_mma[i], 1);
    }
    misc->abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == 0) {
    tmem_alloc(&misc->tmem_base, 128 <= R ? 128 : 64);
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc->tmem_base;
  constexpr uint32_t IDESC = idesc_f16(128, R, 1, 1);
  uint32_t ph_in[2] = {0, 0}, ph_mma[2] = {0, 0};
  int used[2] = {0, 0};   // MMAs were issued on buffer i and not yet waited for
  bool ok = true;
  // job j of the CTA: (tile, layer in group); buffer j % 2
  auto issue_load = [&](long long x, int li, int buf) {
    const int c = (int)(x % nC);
    const long long y = x / nC;
    const int hkv = (int)(y % Hkv), grp = (int)((y / Hkv) % NG), b = (int)(y / ((long long)Hkv * NG));
    const int l = grp * G + li;
    unsigned char* bb = smem + Lay::OFF_BUF + buf * Lay::BUF;
    mbar_expect_tx(&misc->bar_in[buf], (uint32_t)(2 * 16384 + 2 * R * 128));
    const int krow = (int)((((long long)b * L + l) * Hkv + hkv) * N + (long long)c * C);
    for (int ks = 0; ks < 2; ++ks) {
      tma_load_2d(bb + ks * 16384, &tmK, &misc->bar_in[buf], ks * 64, krow);
      tma_load_2d(bb + 2 * 16384 + ks * R * 128, &tmB, &misc->bar_in[buf], ks * 64, (l * Hkv + hkv) * R);
    }
  };
  const long long jobs = (x1 - x0) * G;
  if (tid == 0 && jobs > 0) issue_load(x0, 0, 0);
  for (long long j = 0; ok && j < jobs; ++j) {
    const long long x = x0 + j / G;
    const int li = (int)(j % G), buf = (int)(j & 1);
    if (tid == 0) {
      // the next job's slabs go to the other buffer once the MMAs that read it are done
      if (j + 1 < jobs) {
        const int nb = buf ^ 1;
        if (used[nb]) {
          ok = mbar_wait(&misc->bar_mma[nb], ph_mma[nb], abort_flag, err, ERR_TIMEOUT);
          ph_mma[nb] ^= 1;
          used[nb] = 0;
        }
        if (ok) issue_load(x0 + (j + 1) / G, (int)((j + 1) % G), nb);
      }
      if (ok) ok = mbar_wait(&misc->bar_in[buf], ph_in[buf], abort_flag, err, ERR_TIMEOUT);
      ph_in[buf] ^= 1;
      if (ok) {
        tc_fence_after();
        const unsigned char* bb = smem + Lay::OFF_BUF + buf * Lay::BUF;
        const uint64_t dK = smem_desc(smem_u32(bb), 16, 1024, 2);
        const uint64_t dB = smem_desc(smem_u32(bb + 2 * 16384), 16, 1024, 2);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const int ks = kk >> 2;
          mma_ss(tmem, dK + (uint64_t)((ks * 16384 + (kk & 3) * 32) >> 4),
                 dB + (uint64_t)((ks * R * 128 + (kk & 3) * 32) >> 4), IDESC, (li > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&misc->bar_mma[buf]);
        used[buf] = 1;
      }
    }
    if (!__syncthreads_and(ok)) break;   // every thread leaves at the same point
    if (li != G - 1) continue;
    // the tile is complete: its last MMAs, then the epilogue
    if (tid == 0) {
      ok = mbar_wait(&misc->bar_mma[buf], ph_mma[buf], abort_flag, err, ERR_TIMEOUT);
      ph_mma[buf] ^= 1;
      used[buf] = 0;
    }
    if (!__syncthreads_and(ok)) break;
    tc_fence_after();
    const int c = (int)(x % nC);
    const long long y = x / nC;
    const int hkv = (int)(y % Hkv), grp = (int)((y / Hkv) % NG), b = (int)(y / ((long long)Hkv * NG));
    const size_t row0 = (((size_t)b * NG + grp) * Hkv + hkv) * N + (size_t)c * C;
    const int t = tid;   // token row of the tile = TMEM lane
    const float inv_g = 1.f / (float)G;
    float amax = 0.f;
    if (I8) {   // the row's largest |a| first
#pragma unroll
      for (int q = 0; q < R / 32; ++q) {
        uint32_t v[32];
        tmem_ld32(tmem + ((uint32_t)(32 * warp) << 16) + q * 32, v);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 32; ++k) amax = fmaxf(amax, fabsf(__uint_as_float(v[k]) * inv_g));
      }
    }
#pragma unroll
    for (int q = 0; q < R / 32; ++q) {
      uint32_t v[32];
      tmem_ld32(tmem + ((uint32_t)(32 * warp) << 16) + q * 32, v);
      tmem_wait_ld();
#pragma unroll
      for (int k8 = 0; k8 < 4; ++k8) {
        float x8[8], deq[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) x8[k] = __uint_as_float(v[k8 * 8 + k]) * inv_g;
        const int col = q * 32 + k8 * 8;
        if (I8) {
          __half sh;
          uint2 codes;
          quantize8(x8, amax, &sh, &codes, deq);
          *reinterpret_cast<uint2*>(static_cast<int8_t*>(coeff) + (row0 + t) * R + col) = codes;
          if (col == 0) coeff_scale[row0 + t] = sh;
        } else {
          const uint4 p = pack_bf16x8(x8);
          *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(coeff) + (row0 + t) * R + col) = p;
          const uint32_t pw[4] = {p.x, p.y, p.z, p.w};
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            deq[2 * h] = __uint_as_float(pw[h] << 16);
            deq[2 * h + 1] = __uint_as_float(pw[h] & 0xffff0000u);
          }
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) rows[t * R + ((col + k + t) % R)] = deq[k];   // rotated: no bank conflicts
      }
    }
    tc_fence_before();
    __syncthreads();
    for (int rr = tid; rr < R; rr += 128) {
      float sum = 0.f;
      for (int t2 = 0; t2 < C; ++t2) sum += rows[t2 * R + ((rr + t2) % R)];
      summary[((((size_t)b * NG + grp) * Hkv + hkv) * nC + c) * R + rr] = __float2bfloat16_rn(sum / (float)C);
    }
    __syncthreads();
  }
  // let every copy and MMA this CTA started finish before shared memory and TMEM go away
  if (tid == 0) {
    volatile int never = 0;
    for (int i = 0; i < 2; ++i)
      if (used[i]) mbar_wait(&misc->bar_mma[i], ph_mma[i], &never, err, ERR_TIMEOUT);
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 128 <= R ? 128 : 64);
  }
}

// 2-D tensor map over a row-major [rows][inner] 16-bit array, boxes of 64 x box_rows elements
// in the 128-byte swizzle layout.
bool enc_make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint32_t box_rows) {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return false;
    fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

__global__ void to_half_kernel(const __nv_bfloat16* __restrict__ src, __half* __restrict__ dst, size_t n) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
    dst[i] = __float2half_rn(__bfloat162float(src[i]));
}

// Workspace pieces (256-byte aligned, in this order).
struct EncWs {
  float* w1f_t;            // [L][Hkv][r][h] fp32 W1'
  __nv_bfloat16* w1f_tc;   // [L][Hkv][h][r] W1'/2 (tensor-core path): bf16, fp16 for the int8 store
  __half* w2h;             // [L][Hkv][d][h] fp16 W2 (tensor-core path)
  float* norms;            // [units][N]
  uint8_t* flags;          // [units][N]
  uint32_t* err;           // device error word of the tensor-core kernels
};

// With folds_given the caller supplies both W1' folds, so their regions are left out (the
// pointers stay null until launch_encode points them at the caller's arrays).
EncWs carve(const Geom& g, void* workspace, size_t* bytes, bool folds_given) {
  auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
  const size_t units = (size_t)g.B * g.L * g.Hkv, lh = (size_t)g.L * g.Hkv;
  size_t off = 0;
  auto take = [&](size_t n) {
    unsigned char* p = static_cast<unsigned char*>(workspace) + off;
    off += al(n);
    return p;
  };
  EncWs w;
  w.w1f_t = folds_given ? nullptr : reinterpret_cast<float*>(take(lh * g.r * g.h * 4));
  w.w1f_tc = folds_given ? nullptr : reinterpret_cast<__nv_bfloat16*>(take(lh * g.h * g.r * 2));
  w.w2h = reinterpret_cast<__half*>(take(lh * g.d * g.h * 2));
  w.norms = reinterpret_cast<float*>(take(units * g.N * 4));
  w.flags = take(units * g.N);
  w.err = reinterpret_cast<uint32_t*>(take(4));
  if (bytes) *bytes = off;
  return w;
}

// -------------------------------------- tensor-core coefficients, bases resident (G <= 4)
// The same projection with the group's G bases kept in shared memory for as long as the
// tiles share their (group, KV head), a ring of KST key stages fed ahead of the MMAs, and two
// TMEM accumulators, so that a tile's epilogue (warps 0-3: thread = token row; its stored
// row, and the chunk summary as butterfly sums over the warp plus shared-memory atomics over
// the four warps) overlaps the next tile's MMAs (issued by warp 4).
template <int R>
struct EncCoeff2Layout {
  static constexpr int KST = 3;
  static constexpr int K_BYTES = 2 * 16384;   // 128 tokens x 128 dims, two 64-dim slabs
  static constexpr int B_BYTES = 2 * R * 128;  // R basis rows x 128 dims, two slabs
  static constexpr int OFF_B = 0;              // bases of the group's layers (up to 4)
  static constexpr int OFF_K = OFF_B + 4 * B_BYTES;
  static constexpr int OFF_RED = OFF_K + KST * K_BYTES;   // float [R]: the summary's sums
  static constexpr int OFF_MISC = OFF_RED + R * 4;
  static constexpr int SMEM = OFF_MISC + 192 + 1024;
  static_assert(SMEM <= 227 * 1024, "shared memory");
};

struct EncCoeff2Misc {
  uint64_t b_full, drain, k_full[4], k_empty[4], d_full[2], acc_free[2];
  uint32_t tmem_base;
  int abort_flag;
};

// every thread of the 128-thread named barrier `id` learns whether all of them passed `p`
__device__ __forceinline__ bool named_bar_and(int id, int nthreads, bool p) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred a, b;\n\t"
      "setp.ne.u32 a, %1, 0;\n\t"
      "bar.red.and.pred b, %2, %3, a;\n\t"
      "selp.u32 %0, 1, 0, b;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)p), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}

template <int R, bool I8>
__global__ void __launch_bounds__(160, 1)
enc_coeff_tc2_kernel(int B, int L, int G, int Hkv, int N, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmB, void* __restrict__ coeff,
                     __half* __restrict__ coeff_scale, __nv_bfloat16* __restrict__ summary, uint32_t* err) {
  using namespace tc;
  using Lay = EncCoeff2Layout<R>;
  constexpr int C = 128, KST = Lay::KST;
  extern __shared__ unsigned char encc2_smem_dyn[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(encc2_smem_dyn) + 1023) & ~uintptr_t(1023));
  EncCoeff2Misc* misc = reinterpret_cast<EncCoeff2Misc*>(smem + Lay::OFF_MISC);
  float* red = reinterpret_cast<float*>(smem + Lay::OFF_RED);
  volatile int* abort_flag = &misc->abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nC = N / C, NG = L / G;
  const long long total = (long long)B * NG * Hkv * nC;
  const long long x0 = total * blockIdx.x / gridDim.x, x1 = total * (blockIdx.x + 1) / gridDim.x;
  const long long ntile = x1 - x0;
  if (tid == 0) {
    mbar_init(&misc->b_full, 1);
    mbar_init(&misc->drain, 1);
    for (int s = 0; s < KST; ++s) {
      mbar_init(&misc->k_full[s], 1);
      mbar_init(&misc->k_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&misc->d_full[s], 1);
      mbar_init(&misc->acc_free[s], 4);
    }
    misc->abort_flag = 0;
    mbar_init_fence();
  }
  for (int r = tid; r < R; r += blockDim.x) red[r] = 0.f;
  if (warp == 4) {
    tmem_alloc(&misc->tmem_base, 2 * R);
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc->tmem_base;
  // tile x -> (b, group, KV head, chunk), chunk fastest
  auto tile_of = [&](long long x, int& b, int& grp, int& hkv, int& c) {
    c = (int)(x % nC);
    const long long y = x / nC;
    hkv = (int)(y % Hkv);
    grp = (int)((y / Hkv) % NG);
    b = (int)(y / ((long long)Hkv * NG));
  };

  if (warp == 4) {
    // ============================================================ copies and MMAs
    const bool leader = elect_one();
    constexpr uint32_t IDESC = idesc_f16(128, R, 1, 1);   // keys (bf16) x basis (bf16), both K-major
    const long long jobs = ntile * G;                     // job j: tile j / G, layer j % G
    auto wait_all = [&](uint64_t* bar, uint32_t par, volatile int* flag) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, par, flag, err, ERR_TIMEOUT));
    };
    auto issue_k = [&](long long j) {
      int b, grp, hkv, c;
      tile_of(x0 + j / G, b, grp, hkv, c);
      const int l = grp * G + (int)(j % G);
      const int st = (int)(j % KST);
      const int krow = (int)((((long long)b * L + l) * Hkv + hkv) * N + (long long)c * C);
      if (leader) {
        mbar_expect_tx(&misc->k_full[st], (uint32_t)Lay::K_BYTES);
        for (int ks = 0; ks < 2; ++ks)
          tma_load_2d(smem + Lay::OFF_K + st * Lay::K_BYTES + ks * 16384, &tmK, &misc->k_full[st], ks * 64, krow);
      }
      __syncwarp();
    };
    uint32_t ph_b = 0, ph_d = 0;
    bool ok = true, b_pending = false;
    long long k_issued = 0, k_waited = 0;
    auto load_b = [&](long long i) -> bool {   // the bases of tile i's group layers and KV head
      int b, grp, hkv, c;
      tile_of(x0 + i, b, grp, hkv, c);
      b_pending = true;
      if (leader) {
        mbar_expect_tx(&misc->b_full, (uint32_t)(G * Lay::B_BYTES));
        for (int li = 0; li < G; ++li)
          for (int ks = 0; ks < 2; ++ks)
            tma_load_2d(smem + Lay::OFF_B + li * Lay::B_BYTES + ks * R * 128, &tmB, &misc->b_full, ks * 64,
                        ((grp * G + li) * Hkv + hkv) * R);
      }
      __syncwarp();
      if (!wait_all(&misc->b_full, ph_b, abort_flag)) return false;
      ph_b ^= 1;
      b_pending = false;
      return true;
    };
    auto bseg = [&](long long i) {
      int b, grp, hkv, c;
      tile_of(x0 + i, b, grp, hkv, c);
      return grp * Hkv + hkv;
    };
    auto drain = [&](volatile int* flag) -> bool {
      if (leader) mma_commit(&misc->drain);
      __syncwarp();
      const bool r = wait_all(&misc->drain, ph_d, flag);
      ph_d ^= 1;
      return r;
    };
    if (jobs > 0) {
      for (long long j = 0; j < KST && j < jobs; ++j) issue_k(j);
      k_issued = jobs < KST ? jobs : KST;
      int cur_b = bseg(0);
      ok = load_b(0);
      for (long long j = 0; ok && j < jobs; ++j) {
        const long long i = j / G;
        const int li = (int)(j % G), st = (int)(j % KST), acc = (int)(i & 1);
        if (li == 0 && i > 0 && bseg(i) != cur_b) {   // a new (group, KV head): its bases
          if (!(ok = drain(abort_flag))) break;
          cur_b = bseg(i);
          if (!(ok = load_b(i))) break;
        }
        if (!(ok = wait_all(&misc->k_full[st], (uint32_t)((j / KST) & 1), abort_flag))) break;
        k_waited = j + 1;
        if (li == 0 && i >= 2 && !(ok = wait_all(&misc->acc_free[acc], (uint32_t)(((i >> 1) - 1) & 1), abort_flag)))
          break;
        if (leader) {
          tc_fence_after();
          const uint64_t dK = smem_desc(smem_u32(smem + Lay::OFF_K + st * Lay::K_BYTES), 16, 1024, 2);
          const uint64_t dB = smem_desc(smem_u32(smem + Lay::OFF_B + li * Lay::B_BYTES), 16, 1024, 2);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const int ks = kk >> 2;
            mma_ss(tmem + acc * R, dK + (uint64_t)((ks * 16384 + (kk & 3) * 32) >> 4),
                   dB + (uint64_t)((ks * R * 128 + (kk & 3) * 32) >> 4), IDESC, (li > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&misc->k_empty[st]);
          if (li == G - 1) mma_commit(&misc->d_full[acc]);
        }
        __syncwarp();
        // the stage of job j - 1 (its MMAs are done or nearly so) takes job j - 1 + KST
        const long long jr = j - 1 + KST;
        if (j >= 1 && jr < jobs) {
          const long long jp = j - 1;
          if (!(ok = wait_all(&misc->k_empty[jp % KST], (uint32_t)((jp / KST) & 1), abort_flag))) break;
          issue_k(jr);
          k_issued = jr + 1;
        }
      }
      volatile int never = 0;
      drain(&never);   // every MMA done before TMEM goes
      if (!ok && leader) {
        for (long long j = k_waited; j < k_issued; ++j)
          mbar_wait(&misc->k_full[j % KST], (uint32_t)((j / KST) & 1), &never, err, ERR_TIMEOUT);
        if (b_pending) mbar_wait(&misc->b_full, ph_b, &never, err, ERR_TIMEOUT);
      }
    }
  } else {
    // ============================================================ epilogue (thread = token)
    const int t = tid;
    const uint32_t lane_off = (uint32_t)(32 * warp) << 16;
    const float inv_g = 1.f / (float)G;
    for (long long i = 0; i < ntile; ++i) {
      const int acc = (int)(i & 1);
      bool ok = mbar_wait(&misc->d_full[acc], (uint32_t)((i >> 1) & 1), abort_flag, err, ERR_TIMEOUT);
      if (!named_bar_and(1, 128, ok)) break;   // the four warps leave together
      tc_fence_after();
      int b, grp, hkv, c;
      tile_of(x0 + i, b, grp, hkv, c);
      const size_t row0 = (((size_t)b * NG + grp) * Hkv + hkv) * N + (size_t)c * C;
      const uint32_t tacc = tmem + lane_off + acc * R;
      float amax = 0.f;
      if (I8) {   // the row's largest |a| first
#pragma unroll
        for (int q = 0; q < R / 32; ++q) {
          uint32_t v[32];
          tmem_ld32(tacc + q * 32, v);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) amax = fmaxf(amax, fabsf(__uint_as_float(v[k]) * inv_g));
        }
      }
#pragma unroll
      for (int q = 0; q < R / 32; ++q) {
        uint32_t v[32];
        tmem_ld32(tacc + q * 32, v);
        tmem_wait_ld();
        float dq[32];   // the stored (dequantised) values of columns 32q .. 32q + 31
#pragma unroll
        for (int k8 = 0; k8 < 4; ++k8) {
          float x8[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) x8[k] = __uint_as_float(v[k8 * 8 + k]) * inv_g;
          const int col = q * 32 + k8 * 8;
          if (I8) {
            __half sh;
            uint2 codes;
            quantize8(x8, amax, &sh, &codes, dq + k8 * 8);
            *reinterpret_cast<uint2*>(static_cast<int8_t*>(coeff) + (row0 + t) * R + col) = codes;
            if (col == 0) coeff_scale[row0 + t] = sh;
          } else {
            const uint4 p = pack_bf16x8(x8);
            *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(coeff) + (row0 + t) * R + col) = p;
            const uint32_t pw[4] = {p.x, p.y, p.z, p.w};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              dq[k8 * 8 + 2 * h] = __uint_as_float(pw[h] << 16);
              dq[k8 * 8 + 2 * h + 1] = __uint_as_float(pw[h] & 0xffff0000u);
            }
          }
        }
        // sums over the warp's 32 tokens (transposing butterfly: lane L ends with column
        // 32q + L), then over the four warps in shared memory
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
          const bool up = (lane & o) != 0;
#pragma unroll
          for (int k = 0; k < o; ++k) {
            const float keep = up ? dq[k + o] : dq[k];
            const float give = up ? dq[k] : dq[k + o];
            dq[k] = keep + __shfl_xor_sync(0xffffffffu, give, o);
          }
        }
        atomicAdd(red + q * 32 + lane, dq[0]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&misc->acc_free[acc]);
      named_bar_sync(1, 128);   // every warp's sums are in
      for (int r = t; r < R; r += 128) {
        summary[((((size_t)b * NG + grp) * Hkv + hkv) * nC + c) * R + r] = __float2bfloat16_rn(red[r] / (float)C);
        red[r] = 0.f;
      }
      named_bar_sync(1, 128);   // the sums are reset before the next tile adds to them
    }
  }
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * R);
  }
}

template <int R, int C, bool I8>
cudaError_t launch_encode_t(const Geom& g, int n_res, const void* keys, const void* values,
                            const void* basis, const void* w2, const lowram_encode_dst& dst, const EncWs& w,
                            bool w2h_ready, cudaStream_t s) {
  const int NG = g.L / g.G, nC = g.N / C;
  const size_t units = (size_t)g.B * g.L * g.Hkv;
  dim3 gc(nC, g.Hkv, g.B * NG), gr(nC, g.Hkv, g.B * g.L);
  cudaError_t e;
  int n_sm = 0;
  if ((e = cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, 0)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(w.err, 0, 4, s)) != cudaSuccess) return e;
  if (C == 128) {   // coefficients on tensor cores
    using CL = EncCoeffLayout<R>;
    CUtensorMap tmK, tmB;
    if (!enc_make_map(&tmK, keys, kEncD, (uint64_t)g.B * g.L * g.Hkv * g.N, 128) ||
        !enc_make_map(&tmB, basis, kEncD, (uint64_t)g.L * g.Hkv * R, R))
      return cudaErrorInvalidValue;
    const unsigned cgrid = (unsigned)std::min<size_t>((size_t)n_sm, (size_t)g.B * NG * g.Hkv * nC);
    if (g.G <= 4) {   // the group's bases resident, keys streamed, two accumulators
      using CL2 = EncCoeff2Layout<R>;
      auto kc = enc_coeff_tc2_kernel<R, I8>;
      if ((e = cudaFuncSetAttribute(kc, cudaFuncAttributeMaxDynamicSharedMemorySize, CL2::SMEM)) != cudaSuccess)
        return e;
      kc<<<cgrid, 160, CL2::SMEM, s>>>(g.B, g.L, g.G, g.Hkv, g.N, tmK, tmB, dst.coeff,
                                       static_cast<__half*>(dst.coeff_scale),
                                       static_cast<__nv_bfloat16*>(dst.summary), w.err);
    } else {
      auto kc = enc_coeff_tc_kernel<R, I8>;
      if ((e = cudaFuncSetAttribute(kc, cudaFuncAttributeMaxDynamicSharedMemorySize, CL::SMEM)) != cudaSuccess)
        return e;
      kc<<<cgrid, 128, CL::SMEM, s>>>(g.B, g.L, g.G, g.Hkv, g.N, tmK, tmB, dst.coeff,
                                      static_cast<__half*>(dst.coeff_scale),
                                      static_cast<__nv_bfloat16*>(dst.summary), w.err);
    }
  } else {
    enc_coeff_kernel<R, C, I8><<<gc, kEncThreads, 0, s>>>(
        g.L, g.G, g.Hkv, g.N, static_cast<const __nv_bfloat16*>(keys), static_cast<const __nv_bfloat16*>(basis),
        dst.coeff, static_cast<__half*>(dst.coeff_scale), static_cast<__nv_bfloat16*>(dst.summary));
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (C == 128 || !I8) {   // tensor cores
    using Lay = EncTcLayout<R, C>;
    CUtensorMap tmW1, tmW2, tmA;
    const uint64_t lh = (uint64_t)g.L * g.Hkv;
    if (!enc_make_map(&tmW1, w.w1f_tc, R, lh * kEncH, 128) || !enc_make_map(&tmW2, w.w2h, kEncH, lh * kEncD, 128))
      return cudaErrorInvalidValue;
    if (I8)   // the int8 tiles arrive by plain bulk copies
      tmA = tmW1;
    else if (!enc_make_map(&tmA, dst.coeff, R, (uint64_t)g.B * NG * g.Hkv * g.N, C))
      return cudaErrorInvalidValue;
    if (!w2h_ready)
      to_half_kernel<<<1184, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(w2), w.w2h, (size_t)lh * kEncD * kEncH);
    const unsigned grid = (unsigned)std::min<size_t>((size_t)n_sm, units * nC);
    if (C == 128) {   // tokens as the MMAs' M dimension, two tiles in flight
      using Lay2 = EncTc2Layout<R, I8>;
      auto t1 = enc_resid_tc2_kernel<R, false, I8>;
      auto t2 = enc_resid_tc2_kernel<R, true, I8>;
      if ((e = cudaFuncSetAttribute(t1, cudaFuncAttributeMaxDynamicSharedMemorySize, Lay2::SMEM)) != cudaSuccess) return e;
      if ((e = cudaFuncSetAttribute(t2, cudaFuncAttributeMaxDynamicSharedMemorySize, Lay2::SMEM)) != cudaSuccess) return e;
      t1<<<grid, kEnc2Threads, Lay2::SMEM, s>>>(g.B, g.L, g.G, g.Hkv, g.N, tmW1, tmW2, tmA, dst.coeff,
                                               static_cast<const __half*>(dst.coeff_scale),
                                               static_cast<const __nv_bfloat16*>(values), w.norms, nullptr, nullptr,
                                               nullptr, nullptr, nullptr, w.err);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
      enc_select_kernel<<<(unsigned)units, kSelThreads, (size_t)nC * sizeof(int), s>>>(g.N, C, n_res, w.norms,
                                                                                       w.flags, dst.res_ptr);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
      if (n_res > 0)
        t2<<<grid, kEnc2Threads, Lay2::SMEM, s>>>(g.B, g.L, g.G, g.Hkv, g.N, tmW1, tmW2, tmA, dst.coeff,
                                                 static_cast<const __half*>(dst.coeff_scale),
                                                 static_cast<const __nv_bfloat16*>(values), w.norms, w.flags,
                                                 dst.res_ptr, dst.res_pos, dst.res_val,
                                                 static_cast<__half*>(dst.res_scale), w.err);
      return cudaGetLastError();
    }
    auto k1 = enc_resid_tc_kernel<R, C, false>;
    auto k2 = enc_resid_tc_kernel<R, C, true>;
    if ((e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::SMEM)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::SMEM)) != cudaSuccess) return e;
    k1<<<grid, kEncThreads, Lay::SMEM, s>>>(g.B, g.L, g.G, g.Hkv, g.N, tmW1, tmW2, tmA,
                                            static_cast<const __nv_bfloat16*>(values), w.norms, nullptr, nullptr,
                                            nullptr, nullptr, w.err);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    enc_select_kernel<<<(unsigned)units, kSelThreads, (size_t)nC * sizeof(int), s>>>(g.N, C, n_res, w.norms,
                                                                                     w.flags, dst.res_ptr);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (n_res > 0)
      k2<<<grid, kEncThreads, Lay::SMEM, s>>>(g.B, g.L, g.G, g.Hkv, g.N, tmW1, tmW2, tmA,
                                              static_cast<const __nv_bfloat16*>(values), w.norms, w.flags,
                                              dst.res_ptr, dst.res_pos, static_cast<__nv_bfloat16*>(dst.res_val),
                                              w.err);
    return cudaGetLastError();
  }
  const size_t smem = ResidSmem<R, C>::bytes();
  auto k1 = enc_resid_kernel<R, C, I8, false>;
  auto k2 = enc_resid_kernel<R, C, I8, true>;
  if ((e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess) return e;
  k1<<<gr, kEncThreads, smem, s>>>(g.L, g.G, g.Hkv, g.N, n_res, dst.coeff, static_cast<const __half*>(dst.coeff_scale),
                                   w.w1f_t, static_cast<const __nv_bfloat16*>(w2),
                                   static_cast<const __nv_bfloat16*>(values), w.norms, nullptr, nullptr, nullptr,
                                   nullptr, nullptr);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  enc_select_kernel<<<(unsigned)units, kSelThreads, (size_t)nC * sizeof(int), s>>>(g.N, C, n_res, w.norms, w.flags,
                                                                                   dst.res_ptr);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (n_res > 0)
    k2<<<gr, kEncThreads, smem, s>>>(g.L, g.G, g.Hkv, g.N, n_res, dst.coeff,
                                     static_cast<const __half*>(dst.coeff_scale), w.w1f_t,
                                     static_cast<const __nv_bfloat16*>(w2), static_cast<const __nv_bfloat16*>(values),
                                     w.norms, w.flags, dst.res_ptr, dst.res_pos, dst.res_val,
                                     static_cast<__half*>(dst.res_scale));
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_to_half(const __nv_bfloat16* src, __half* dst, size_t n, cudaStream_t s) {
  to_half_kernel<<<1184, 256, 0, s>>>(src, dst, n);
  return cudaGetLastError();
}

size_t encode_workspace_bytes(const Geom& g, bool folds_given) {
  size_t bytes = 0;
  carve(g, nullptr, &bytes, folds_given);
  return bytes;
}

uint32_t* encode_error_word(const Geom& g, void* workspace, bool folds_given) {
  size_t bytes = 0;
  return carve(g, workspace, &bytes, folds_given).err;
}

cudaError_t launch_encode(const Geom& g, int store, int n_res, const void* keys, const void* values,
                          const void* basis, const void* w1, const void* w2, const lowram_encode_dst& dst,
                          void* workspace, cudaStream_t s) {
  return launch_encode(g, store, n_res, keys, values, basis, w1, w2, dst, workspace, s, nullptr, nullptr, false);
}

cudaError_t launch_encode(const Geom& g, int store, int n_res, const void* keys, const void* values,
                          const void* basis, const void* w1, const void* w2, const lowram_encode_dst& dst,
                          void* workspace, cudaStream_t s, const float* w1f_t, const void* w1f_tc,
                          bool w2h_ready) {
  const bool i8 = store == LOWRAM_STORE_INT8;
  const bool folds_given = w1f_t && w1f_tc;
  EncWs w = carve(g, workspace, nullptr, folds_given);
  if (folds_given) {   // the caller's folds: fp32, and W1'/2 in bf16 (native) or fp16 (int8 store)
    w.w1f_t = const_cast<float*>(w1f_t);
    w.w1f_tc = static_cast<__nv_bfloat16*>(const_cast<void*>(w1f_tc));
  } else {
    CacheBuffers cb{};
    cb.w1 = w1;
    cb.basis = basis;
    cudaError_t e = launch_fold(g, cb, LOWRAM_BF16, i8 ? LOWRAM_STORE_INT8 : LOWRAM_STORE_NATIVE, w.w1f_t,
                                w.w1f_tc, s);
    if (e != cudaSuccess) return e;
  }
#define LOWRAM_ENC_CASE(RR, CC)                                                                          \
  if (g.r == RR && g.C == CC)                                                                            \
    return i8 ? launch_encode_t<RR, CC, true>(g, n_res, keys, values, basis, w2, dst, w, w2h_ready, s)   \
              : launch_encode_t<RR, CC, false>(g, n_res, keys, values, basis, w2, dst, w, w2h_ready, s);
  LOWRAM_ENC_CASE(128, 128)
  LOWRAM_ENC_CASE(128, 64)
  LOWRAM_ENC_CASE(64, 128)
  LOWRAM_ENC_CASE(64, 64)
#undef LOWRAM_ENC_CASE
  return cudaErrorNotSupported;
}

}  // namespace lowram
