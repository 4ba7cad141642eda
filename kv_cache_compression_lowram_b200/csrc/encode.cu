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
// All CUDA-core fp32 arithmetic from bf16 inputs (register-tiled, operands staged in shared
// memory); the tensor-core form of the two contractions is future work.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "lowram_internal.cuh"

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

template <int R, int C, bool I8>
cudaError_t launch_encode_t(const Geom& g, int n_res, const void* keys, const void* values,
                            const void* basis, const void* w2, const lowram_encode_dst& dst,
                            const float* w1f_t, float* norms, uint8_t* flags, cudaStream_t s) {
  const int NG = g.L / g.G, nC = g.N / C;
  dim3 gc(nC, g.Hkv, g.B * NG), gr(nC, g.Hkv, g.B * g.L);
  enc_coeff_kernel<R, C, I8><<<gc, kEncThreads, 0, s>>>(
      g.L, g.G, g.Hkv, g.N, static_cast<const __nv_bfloat16*>(keys), static_cast<const __nv_bfloat16*>(basis),
      dst.coeff, static_cast<__half*>(dst.coeff_scale), static_cast<__nv_bfloat16*>(dst.summary));
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t smem = ResidSmem<R, C>::bytes();
  auto k1 = enc_resid_kernel<R, C, I8, false>;
  auto k2 = enc_resid_kernel<R, C, I8, true>;
  if ((e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess) return e;
  k1<<<gr, kEncThreads, smem, s>>>(g.L, g.G, g.Hkv, g.N, n_res, dst.coeff, static_cast<const __half*>(dst.coeff_scale),
                                   w1f_t, static_cast<const __nv_bfloat16*>(w2),
                                   static_cast<const __nv_bfloat16*>(values), norms, nullptr, nullptr, nullptr,
                                   nullptr, nullptr);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const size_t units = (size_t)g.B * g.L * g.Hkv;
  enc_select_kernel<<<(unsigned)units, kSelThreads, (size_t)nC * sizeof(int), s>>>(g.N, C, n_res, norms, flags,
                                                                                   dst.res_ptr);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (n_res > 0)
    k2<<<gr, kEncThreads, smem, s>>>(g.L, g.G, g.Hkv, g.N, n_res, dst.coeff,
                                     static_cast<const __half*>(dst.coeff_scale), w1f_t,
                                     static_cast<const __nv_bfloat16*>(w2), static_cast<const __nv_bfloat16*>(values),
                                     norms, flags, dst.res_ptr, dst.res_pos, dst.res_val,
                                     static_cast<__half*>(dst.res_scale));
  return cudaGetLastError();
}

}  // namespace

size_t encode_workspace_bytes(const Geom& g) {
  const size_t units = (size_t)g.B * g.L * g.Hkv;
  auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
  return al((size_t)g.L * g.Hkv * g.r * g.h * 4) + al(units * g.N * 4) + al(units * g.N);
}

cudaError_t launch_encode(const Geom& g, int store, int n_res, const void* keys, const void* values,
                          const void* basis, const void* w1, const void* w2, const lowram_encode_dst& dst,
                          void* workspace, cudaStream_t s) {
  auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
  const size_t units = (size_t)g.B * g.L * g.Hkv;
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  float* w1f_t = reinterpret_cast<float*>(ws);
  float* norms = reinterpret_cast<float*>(ws + al((size_t)g.L * g.Hkv * g.r * g.h * 4));
  uint8_t* flags = reinterpret_cast<uint8_t*>(ws + al((size_t)g.L * g.Hkv * g.r * g.h * 4) + al(units * g.N * 4));
  CacheBuffers cb{};
  cb.w1 = w1;
  cb.basis = basis;
  cudaError_t e = launch_fold(g, cb, LOWRAM_BF16, LOWRAM_STORE_NATIVE, w1f_t, nullptr, s);
  if (e != cudaSuccess) return e;
  const bool i8 = store == LOWRAM_STORE_INT8;
#define LOWRAM_ENC_CASE(RR, CC)                                                                      \
  if (g.r == RR && g.C == CC)                                                                        \
    return i8 ? launch_encode_t<RR, CC, true>(g, n_res, keys, values, basis, w2, dst, w1f_t, norms, flags, s) \
              : launch_encode_t<RR, CC, false>(g, n_res, keys, values, basis, w2, dst, w1f_t, norms, flags, s);
  LOWRAM_ENC_CASE(128, 128)
  LOWRAM_ENC_CASE(128, 64)
  LOWRAM_ENC_CASE(64, 128)
  LOWRAM_ENC_CASE(64, 64)
#undef LOWRAM_ENC_CASE
  return cudaErrorNotSupported;
}

}  // namespace lowram
