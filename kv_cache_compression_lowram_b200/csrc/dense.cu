// Dense (uncompressed) decode attention over a bf16 KV cache: the baseline the compressed
// path is compared with.  Every cached token is attended:
//     o_j = softmax_t(q_j . k_t / sqrt(d)) v_t         ("OjaKV", section 3, attention)
// and the cache costs M_KV = 2 L H_kv d N s bytes per sequence ("LowRAM Compresses KV Cache
// Asymmetrically", section "Core Mechanism").
//
// One CTA per (sequence, layer, KV head) streams its K and V once, in blocks of 256 tokens:
// thread t scores token t against every query head of the unit (16-byte loads of its key
// row), the block's softmax update is a warp reduction per head, and thread (head, dim pair)
// accumulates P.V with coalesced 4-byte loads of V.  The kernel is bound by HBM.
#include "lowram_internal.cuh"

namespace lowram {
namespace {

constexpr int kThreads = 256;
constexpr int kBlock = 256;   // tokens per block (one per thread)
constexpr int kMaxGD = 16;    // query heads per KV head

__global__ void __launch_bounds__(kThreads)
dense_kernel(int B, int L, int Hkv, int Hq, int d, long long S, const __nv_bfloat16* __restrict__ K,
             const __nv_bfloat16* __restrict__ V, const __nv_bfloat16* __restrict__ q,
             __nv_bfloat16* __restrict__ out, float scale_log2) {
  extern __shared__ __align__(16) float sm[];
  const int g = Hq / Hkv;
  float* qs = sm;                       // [g][d]
  float* p = qs + g * d;                // [g][kBlock]
  float* acc = p + g * kBlock;          // [g][d]
  float* stat = acc + g * d;            // m[g], l[g], alpha[g]
  const int u = blockIdx.x;             // unit = ((l * B) + b) * Hkv + hkv
  const int hkv = u % Hkv;
  const int b = (u / Hkv) % B;
  const int l = u / (Hkv * B);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarp = blockDim.x >> 5;
  const size_t qoff = ((size_t)(l * B + b) * Hq + (size_t)hkv * g) * d;
  for (int i = tid; i < g * d; i += blockDim.x) {
    qs[i] = __bfloat162float(q[qoff + i]);
    acc[i] = 0.f;
  }
  if (tid < g) {
    stat[tid] = -INFINITY;
    stat[g + tid] = 0.f;
  }
  __syncthreads();
  const size_t kvoff = (((size_t)b * L + l) * Hkv + hkv) * (size_t)S * d;
  const __nv_bfloat16* Ku = K + kvoff;
  const __nv_bfloat16* Vu = V + kvoff;
  for (long long t0 = 0; t0 < S; t0 += kBlock) {
    const int nb = (int)(S - t0 < kBlock ? S - t0 : kBlock);
    if (tid < nb) {
      const uint4* row = reinterpret_cast<const uint4*>(Ku + (size_t)(t0 + tid) * d);
      float a[kMaxGD];
#pragma unroll
      for (int j = 0; j < kMaxGD; ++j) a[j] = 0.f;
      for (int e = 0; e < d / 8; ++e) {
        const uint4 w4 = __ldg(row + e);
        const uint32_t w[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float k0 = __uint_as_float(w[i] << 16), k1 = __uint_as_float(w[i] & 0xffff0000u);
#pragma unroll
          for (int j = 0; j < kMaxGD; ++j) {
            if (j < g) {
              a[j] = fmaf(k0, qs[j * d + e * 8 + 2 * i], a[j]);
              a[j] = fmaf(k1, qs[j * d + e * 8 + 2 * i + 1], a[j]);
            }
          }
        }
      }
#pragma unroll
      for (int j = 0; j < kMaxGD; ++j)
        if (j < g) p[j * kBlock + tid] = a[j] * scale_log2;
    }
    __syncthreads();
    for (int j = warp; j < g; j += nwarp) {
      float m = -INFINITY;
      for (int t = lane; t < nb; t += 32) m = fmaxf(m, p[j * kBlock + t]);
      m = warp_max(m);
      const float mnew = fmaxf(stat[j], m);
      float s = 0.f;
      for (int t = lane; t < nb; t += 32) {
        const float e = exp2f(p[j * kBlock + t] - mnew);
        p[j * kBlock + t] = e;
        s += e;
      }
      s = warp_sum(s);
      if (lane == 0) {
        const float a = exp2f(stat[j] - mnew);
        stat[2 * g + j] = a;
        stat[g + j] = stat[g + j] * a + s;
        stat[j] = mnew;
      }
    }
    __syncthreads();
    for (int item = tid; item < g * (d / 2); item += blockDim.x) {
      const int j = item / (d / 2), dp = item % (d / 2);
      const float* pj = p + j * kBlock;
      const uint32_t* vcol = reinterpret_cast<const uint32_t*>(Vu + (size_t)t0 * d) + dp;
      float a0 = 0.f, a1 = 0.f, c0 = 0.f, c1 = 0.f;
      int t = 0;
      for (; t + 2 <= nb; t += 2) {
        const uint32_t v0 = __ldg(vcol + (size_t)t * (d / 2));
        const uint32_t v1 = __ldg(vcol + (size_t)(t + 1) * (d / 2));
        a0 = fmaf(pj[t], __uint_as_float(v0 << 16), a0);
        a1 = fmaf(pj[t], __uint_as_float(v0 & 0xffff0000u), a1);
        c0 = fmaf(pj[t + 1], __uint_as_float(v1 << 16), c0);
        c1 = fmaf(pj[t + 1], __uint_as_float(v1 & 0xffff0000u), c1);
      }
      if (t < nb) {
        const uint32_t v0 = __ldg(vcol + (size_t)t * (d / 2));
        a0 = fmaf(pj[t], __uint_as_float(v0 << 16), a0);
        a1 = fmaf(pj[t], __uint_as_float(v0 & 0xffff0000u), a1);
      }
      const float al = stat[2 * g + j];
      acc[j * d + 2 * dp] = acc[j * d + 2 * dp] * al + a0 + c0;
      acc[j * d + 2 * dp + 1] = acc[j * d + 2 * dp + 1] * al + a1 + c1;
    }
    __syncthreads();
  }
  __nv_bfloat16* o = out + qoff;
  for (int i = tid; i < g * d; i += blockDim.x) o[i] = __float2bfloat16_rn(acc[i] / stat[g + i / d]);
}

}  // namespace
}  // namespace lowram

extern "C" lowram_status lowram_dense_decode_attn(int32_t batch, int32_t n_layers, int32_t n_kv_heads,
                                                  int32_t n_q_heads, int32_t head_dim, int64_t seq_len,
                                                  const void* k, const void* v, const void* q, void* out,
                                                  lowram_stream stream) {
  using namespace lowram;
  if (batch < 1 || n_layers < 1 || n_kv_heads < 1 || n_q_heads < 1 || seq_len < 1 ||
      n_q_heads % n_kv_heads || n_q_heads / n_kv_heads > kMaxGD || head_dim < 8 ||
      head_dim % 8 || head_dim > kMaxD)
    return LOWRAM_EINVAL;
  if (!k || !v || !q || !out || (reinterpret_cast<uintptr_t>(k) & 15) || (reinterpret_cast<uintptr_t>(v) & 15))
    return LOWRAM_EINVAL;
  const long long units = (long long)batch * n_layers * n_kv_heads;
  if (units > 0x7fffffffLL) return LOWRAM_EINVAL;
  const int g = n_q_heads / n_kv_heads;
  const size_t smem = sizeof(float) * ((size_t)g * head_dim * 2 + (size_t)g * kBlock + 3 * g);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaFuncSetAttribute(dense_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return LOWRAM_ECUDA;
  dense_kernel<<<(unsigned)units, kThreads, smem, s>>>(
      batch, n_layers, n_kv_heads, n_q_heads, head_dim, seq_len, static_cast<const __nv_bfloat16*>(k),
      static_cast<const __nv_bfloat16*>(v), static_cast<const __nv_bfloat16*>(q),
      static_cast<__nv_bfloat16*>(out), 1.4426950408889634f / sqrtf((float)head_dim));
  return cudaGetLastError() == cudaSuccess ? LOWRAM_OK : LOWRAM_ECUDA;
}
