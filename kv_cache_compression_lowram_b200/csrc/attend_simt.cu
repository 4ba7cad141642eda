// Steps 3-5 on CUDA cores: rebuild the selected chunks and attend over them.
//
// For every token t of a selected chunk (coefficient row a_t, int8 scale sigma_t or 1):
//   score   l_jt = sigma_t * qt_j . a_t            (qt_j = B_l q_j * log2(e)/sqrt(d): the
//                                                   low-rank form of q_j . khat_t / sqrt(d))
//   hidden  h_t  = silu(sigma_t * W1' a_t)          (W1' = W1 B_l^T, exact fold of W1 khat_t)
//   softmax partials over the chunk tokens, then
//   accH_j += sum_t p_jt h_t,  accD_j += sum_t p_jt rho_t delta_t (flagged tokens only).
// The second predictor layer is applied once per unit in the combine step:
// sum_t p_t (W2 h_t + delta_t) = W2 (sum_t p_t h_t) + sum_t p_t delta_t.
// Key rebuild: "LowRAM Compresses KV Cache Asymmetrically", section "Cross-Layer Low-Rank Key
// Compression"; values: same page, section "Core Mechanism" (Vhat = f(K), delta = V - Vhat
// for the worst tokens); attention: "OjaKV", section 3.
//
// This path serves every shape (and is the only one for fp32 caches).  Each CTA walks a
// contiguous range of (unit, selected chunk) tiles and writes one partial record per unit
// piece it touched.
#include "lowram_internal.cuh"

namespace lowram {
namespace {

constexpr int kThreads = 256;
constexpr int kTB = 64;   // tokens per sub-block
constexpr int kTT = 16;   // tokens per register block of the hidden-layer loop

__device__ __forceinline__ float silu_f(float x) { return x / (1.f + __expf(-x)); }

template <typename T, bool INT8>
__global__ void __launch_bounds__(kThreads)
attend_simt_kernel(Geom g, CacheBuffers cb, Scratch sc, const float* __restrict__ w1f_t, int w1f_layer0) {
  extern __shared__ __align__(16) float sm[];
  const int rp = g.r + 1;                       // padded row (bank-conflict free)
  float* a_s = sm;                              // [kTB][rp]
  float* qt_s = a_s + kTB * rp;                 // [g][r]
  float* p_s = qt_s + g.g * g.r;                // [g][kTB]
  float* accH = p_s + g.g * kTB;                // [g][h]
  float* accD = accH + g.g * g.h;               // [g][d]
  float* mrun = accD + g.g * g.d;               // [g]
  float* lrun = mrun + g.g;                     // [g]
  float* alpha = lrun + g.g;                    // [g]

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarp = blockDim.x >> 5;
  const long long total = (long long)g.U * g.k;
  const int c = blockIdx.x;
  const long long x0 = tile_begin(total, g.P, c), x1 = tile_begin(total, g.P, c + 1);
  const int NG = g.L / g.G;

  int cur = -1;
  for (long long x = x0; x <= x1; ++x) {
    const int u = x < x1 ? (int)(x / g.k) : -1;
    if (u != cur) {
      if (cur >= 0) {  // flush the finished piece of unit `cur`
        float* rec = sc.part + (size_t)(cur + c) * g.rec_stride;
        for (int i = tid; i < g.g; i += blockDim.x) {
          rec[i] = mrun[i];
          rec[g.g + i] = lrun[i];
        }
        for (int i = tid; i < g.g * g.h; i += blockDim.x) rec[2 * g.g + i] = accH[i];
        for (int i = tid; i < g.g * g.d; i += blockDim.x) rec[2 * g.g + g.g * g.h + i] = accD[i];
        __syncthreads();
      }
      if (u < 0) break;
      cur = u;
      for (int i = tid; i < g.g * g.r; i += blockDim.x) qt_s[i] = sc.qt[(size_t)u * g.g * g.r + i];
      for (int i = tid; i < g.g * g.h; i += blockDim.x) accH[i] = 0.f;
      for (int i = tid; i < g.g * g.d; i += blockDim.x) accD[i] = 0.f;
      if (tid < g.g) {
        mrun[tid] = -INFINITY;
        lrun[tid] = 0.f;
      }
      __syncthreads();
    }
    const Unit un = unit_of(g, u);
    const int l = g.layer0 + un.li;
    const int grp = l / g.G;
    const int slot = sc.sel_slot[x];
    const size_t row0 = ((((size_t)un.b * NG + grp) * g.Hkv + un.hkv) * g.nLs + slot) * g.C;
    const T* coeff = reinterpret_cast<const T*>(cb.coeff);
    const int8_t* coeff8 = reinterpret_cast<const int8_t*>(cb.coeff);
    const float* w1 = w1f_t + ((size_t)(l - w1f_layer0) * g.Hkv + un.hkv) * g.r * g.h;
    const int32_t* rptr = cb.res_ptr + (((size_t)un.b * g.L + l) * g.Hkv + un.hkv) * (g.nLs + 1);
    // a record range outside [0, n_records] (a corrupt CSR table; the caller's own arrays on
    // the allocation-free path are never validated) is clamped and reported, so no record
    // read leaves the arrays
    int rec0 = rptr[slot], rec1 = rptr[slot + 1];
    if (rec0 < 0 || rec1 < rec0 || (long long)rec1 > cb.n_records) {
      if (tid == 0) atomicOr(sc.err, ERR_RES_PTR);
      rec0 = (int)max(0ll, min((long long)rec0, (long long)cb.n_records));
      rec1 = (int)max((long long)rec0, min((long long)rec1, (long long)cb.n_records));
    }

    for (int t0 = 0; t0 < g.C; t0 += kTB) {
      const int nb = min(kTB, g.C - t0);
      // coefficient rows (dequantised)
      for (int i = tid; i < nb * g.r; i += blockDim.x) {
        const int t = i / g.r, rr = i % g.r;
        const size_t row = row0 + t0 + t;
        float v;
        if (INT8) v = (float)coeff8[row * g.r + rr] * __half2float(cb.coeff_scale[row]);
        else v = to_f(coeff[row * g.r + rr]);
        a_s[t * rp + rr] = v;
      }
      __syncthreads();
      // scores (log2 domain)
      for (int i = tid; i < g.g * nb; i += blockDim.x) {
        const int j = i / nb, t = i % nb;
        const float* q = qt_s + j * g.r;
        const float* a = a_s + t * rp;
        float s = 0.f;
        for (int rr = 0; rr < g.r; ++rr) s = fmaf(q[rr], a[rr], s);
        p_s[j * kTB + t] = s;
      }
      __syncthreads();
      // online softmax update per head
      for (int j = warp; j < g.g; j += nwarp) {
        float m = -INFINITY;
        for (int t = lane; t < nb; t += 32) m = fmaxf(m, p_s[j * kTB + t]);
        m = warp_max(m);
        const float mnew = fmaxf(mrun[j], m);
        float s = 0.f;
        for (int t = lane; t < nb; t += 32) {
          const float p = exp2f(p_s[j * kTB + t] - mnew);
          p_s[j * kTB + t] = p;
          s += p;
        }
        s = warp_sum(s);
        if (lane == 0) {
          const float a = exp2f(mrun[j] - mnew);
          alpha[j] = a;
          lrun[j] = lrun[j] * a + s;
          mrun[j] = mnew;
        }
      }
      __syncthreads();
      for (int i = tid; i < g.g * g.h; i += blockDim.x) accH[i] *= alpha[i / g.h];
      for (int i = tid; i < g.g * g.d; i += blockDim.x) accD[i] *= alpha[i / g.d];
      __syncthreads();
      // hidden layer: each thread owns hidden units i
      for (int i = tid; i < g.h; i += blockDim.x) {
        for (int tb = 0; tb < nb; tb += kTT) {
          float pre[kTT];
#pragma unroll
          for (int tt = 0; tt < kTT; ++tt) pre[tt] = 0.f;
          for (int rr = 0; rr < g.r; ++rr) {
            const float w = __ldg(w1 + (size_t)rr * g.h + i);
#pragma unroll
            for (int tt = 0; tt < kTT; ++tt)
              if (tb + tt < nb) pre[tt] = fmaf(w, a_s[(tb + tt) * rp + rr], pre[tt]);
          }
#pragma unroll
          for (int tt = 0; tt < kTT; ++tt) {
            if (tb + tt < nb) {
              const float hv = silu_f(pre[tt]);
              for (int j = 0; j < g.g; ++j) accH[j * g.h + i] = fmaf(p_s[j * kTB + tb + tt], hv, accH[j * g.h + i]);
            }
          }
        }
      }
      // residual rows of the flagged tokens in this sub-block
      for (int i = tid; i < g.g * g.d; i += blockDim.x) {
        const int j = i / g.d, dd = i % g.d;
        float a = 0.f;
        for (int rec = rec0; rec < rec1; ++rec) {
          const int pos = (int)cb.res_pos[rec];
          if (pos < t0 || pos >= t0 + nb) continue;
          float dv;
          if (INT8)
            dv = (float)reinterpret_cast<const int8_t*>(cb.res_val)[(size_t)rec * g.d + dd] *
                 __half2float(cb.res_scale[rec]);
          else
            dv = to_f(reinterpret_cast<const T*>(cb.res_val)[(size_t)rec * g.d + dd]);
          a = fmaf(p_s[j * kTB + pos - t0], dv, a);
        }
        accD[i] += a;
      }
      __syncthreads();
    }
  }
}

size_t simt_smem_bytes(const Geom& g) {
  return sizeof(float) * ((size_t)kTB * (g.r + 1) + (size_t)g.g * g.r + (size_t)g.g * kTB +
                          (size_t)g.g * g.h + (size_t)g.g * g.d + 3 * g.g);
}

}  // namespace

cudaError_t launch_attend_simt(const Geom& g, const CacheBuffers& cb, const Scratch& sc,
                               int dtype, int store, const float* w1f_t, int w1f_layer0,
                               cudaStream_t s) {
  const size_t smem = simt_smem_bytes(g);
  if (smem > 227 * 1024) return cudaErrorInvalidConfiguration;
  cudaError_t e;
  if (dtype == LOWRAM_F32) {
    auto k = attend_simt_kernel<float, false>;
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<g.P, kThreads, smem, s>>>(g, cb, sc, w1f_t, w1f_layer0);
  } else if (store == LOWRAM_STORE_INT8) {
    auto k = attend_simt_kernel<__nv_bfloat16, true>;
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<g.P, kThreads, smem, s>>>(g, cb, sc, w1f_t, w1f_layer0);
  } else {
    auto k = attend_simt_kernel<__nv_bfloat16, false>;
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<g.P, kThreads, smem, s>>>(g, cb, sc, w1f_t, w1f_layer0);
  }
  return cudaGetLastError();
}

}  // namespace lowram
