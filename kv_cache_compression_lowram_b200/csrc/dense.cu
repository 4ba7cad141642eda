// Dense (uncompressed) decode attention over a bf16 KV cache: the baseline the compressed
// path is compared with.  Every cached token is attended:
//     o_j = softmax_t(q_j . k_t / sqrt(d)) v_t         ("OjaKV", section 3, attention)
// and the cache costs M_KV = 2 L H_kv d N s bytes per sequence ("LowRAM Compresses KV Cache
// Asymmetrically", section "Core Mechanism").  The kernel streams K and V once, so it is
// bound by HBM bandwidth; at d = 128 it moves 512 bytes per token and query group.
//
// Tensor-core kernel (d = 128, g = Hq/Hkv in {1, 2, 4, 8, 16}, q 16-byte aligned): one CTA
// per (sequence, layer, KV head) walks its tokens in tiles of 128, three tiles in flight:
//   warp 4      TMA producer: the K and V tiles (two 64-column slabs each, 128-byte swizzle;
//               3-D maps [unit][token][dim], so rows past the sequence read as zeros) and
//               the unit's queries,
//   warp 5      MMA issuer + TMEM owner:
//                 S  = K_tile . Q^T   M = 128 tokens, N = 16 query heads (g used), K = d
//                 O  = V_tile^T . P^T M = 128 dims, N = 16 heads, K = 128 tokens (V read
//                                     MN-major as TMA delivers it; P bf16 in shared memory)
//               S and O double-buffered in TMEM, S(i+2) issued behind O(i),
//   warps 0-3   softmax: thread = token of the tile for the scores (online max per head
//               over the tile, P written to shared memory), then thread = output dimension
//               for the fold acc = acc * alpha + O(i-1) of the previous tile.
// Other shapes take a CUDA-core kernel (one CTA per unit, 256-token blocks).
//
// Every wait is bounded: when one runs out the unit's outputs are written as NaN, the
// kernel drains its own copies and MMAs, frees TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "lowram_internal.cuh"
#include "tc_ptx.cuh"

namespace lowram {
namespace {

using namespace tc;

// ============================================================== tensor-core kernel

constexpr int kDD = 128;                    // head dim of the tensor-core kernel
constexpr int kTok = 128;                   // tokens per tile
constexpr int kDStages = 3;
constexpr int kSlab = kTok * 128;           // one 64-column slab of a tile (bytes)
constexpr int kStageBytes = 4 * kSlab;      // K slabs 0,1 then V slabs 0,1
constexpr int kOffQ = kDStages * kStageBytes;
constexpr int kQBytes = 2 * 16 * 128;       // 16 query rows x 128 dims bf16, two slabs
constexpr int kOffP = kOffQ + kQBytes;
constexpr int kPSbo = (kTok / 8) * 128;     // P: no-swizzle K-major, 8-row groups 2048 B apart
constexpr int kPBuf = 2 * kPSbo;            // 16 rows
constexpr int kOffMisc = kOffP + 2 * kPBuf;
constexpr int kDThreads = 192;              // warps 0-3 softmax, 4 producer, 5 MMA
constexpr int kTmemCols = 64;               // S double buffer [0,32), O double buffer [32,64)

struct DenseMisc {
  uint64_t full[kDStages], empty[kDStages];
  uint64_t q_full, s_full[2], p_ready[2], o_full[2], drain;
  float red[2][4][16];                      // per-warp partial max (two tiles in flight)
  uint32_t tmem_base;
  int abort_flag;
};
constexpr int kDenseSmem = kOffMisc + (int)sizeof(DenseMisc) + 1024;   // + alignment slack
static_assert(kOffQ % 1024 == 0 && kOffP % 16 == 0 && kOffMisc % 8 == 0, "operand alignment");
static_assert(kDenseSmem <= 232448, "shared memory per CTA");

__device__ uint32_t g_dense_err;            // bounded-wait timeouts of the tensor-core kernel

__device__ __forceinline__ void tma_load_3d(void* dst, const void* tmap, uint64_t* bar, int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}

// Barrier 1 among the 128 softmax threads that also ORs a predicate over them: every thread
// gets the same answer, so an abort decision taken from it never splits the group.
__device__ __forceinline__ bool softmax_sync_or(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.or.pred p, 1, 128, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v)
      : "memory");
  return r != 0;
}

// Byte offset of element (row n, column k) in a no-swizzle K-major operand of 8 x 16-byte
// core matrices: core matrices 128 B apart along K, 8-row groups sbo apart.
__device__ __forceinline__ uint32_t core_off(int n, int k, int sbo) {
  return (uint32_t)((n >> 3) * sbo + (k >> 3) * 128 + (n & 7) * 16 + (k & 7) * 2);
}

template <int GQ>
__global__ void __launch_bounds__(kDThreads, 1)
dense_tc_kernel(int B, int L, int Hkv, int Hq, long long S, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmQ,
                __nv_bfloat16* __restrict__ out, float scale_log2) {
  extern __shared__ unsigned char smem_dyn[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
  DenseMisc* m = reinterpret_cast<DenseMisc*>(smem + kOffMisc);
  volatile int* abort_flag = &m->abort_flag;
  uint32_t* err = &g_dense_err;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int u = blockIdx.x;                 // ((l * B) + b) * Hkv + hkv
  const int hkv = u % Hkv;
  const int b = (u / Hkv) % B;
  const int l = u / (Hkv * B);
  const int kvu = (b * L + l) * Hkv + hkv;  // unit index of the [B][L][Hkv] K/V layout
  const int qrow = (l * B + b) * Hq + hkv * GQ;
  const int nt = (int)((S + kTok - 1) / kTok);

  if (tid == 0) {
    for (int i = 0; i < kDStages; ++i) {
      mbar_init(&m->full[i], 1);
      mbar_init(&m->empty[i], 1);
    }
    mbar_init(&m->q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&m->s_full[i], 1);
      mbar_init(&m->p_ready[i], 1);
      mbar_init(&m->o_full[i], 1);
    }
    mbar_init(&m->drain, 1);
    m->abort_flag = 0;
    mbar_init_fence();
  }
  // P rows >= GQ stay zero for the whole kernel
  for (int i = tid; i < 2 * kPBuf / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(smem + kOffP)[i] = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
  if (warp == 5) {
    tmem_alloc(&m->tmem_base, kTmemCols);
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = m->tmem_base;

  if (warp == 4) {
    // ============================================================ TMA producer
    const bool leader = elect_one();
    int issued = 0;
    if (leader) {
      mbar_expect_tx(&m->q_full, kQBytes);
      tma_load_2d(smem + kOffQ, &tmQ, &m->q_full, 0, qrow);
      tma_load_2d(smem + kOffQ + kQBytes / 2, &tmQ, &m->q_full, 64, qrow);
    }
    for (int i = 0; i < nt; ++i) {
      const int st = i % kDStages;
      if (i >= kDStages &&
          !__all_sync(0xffffffffu, mbar_wait(&m->empty[st], ((i / kDStages) - 1) & 1, abort_flag, err, 1u)))
        break;
      if (leader) {
        unsigned char* dst = smem + st * kStageBytes;
        mbar_expect_tx(&m->full[st], kStageBytes);
        tma_load_3d(dst, &tmK, &m->full[st], 0, i * kTok, kvu);
        tma_load_3d(dst + kSlab, &tmK, &m->full[st], 64, i * kTok, kvu);
        tma_load_3d(dst + 2 * kSlab, &tmV, &m->full[st], 0, i * kTok, kvu);
        tma_load_3d(dst + 3 * kSlab, &tmV, &m->full[st], 64, i * kTok, kvu);
      }
      __syncwarp();
      issued = i + 1;
    }
    // every copy this CTA started lands before it exits (the last phase of each stage)
    int never = 0;
    for (int i = max(0, issued - kDStages); i < issued; ++i)
      mbar_wait(&m->full[i % kDStages], (i / kDStages) & 1, &never, err, 1u);
    mbar_wait(&m->q_full, 0, &never, err, 1u);
  } else if (warp == 5) {
    // ============================================================ MMA issuer
    const bool leader = elect_one();
    const uint32_t sKV = smem_u32(smem), sQ = smem_u32(smem + kOffQ), sP = smem_u32(smem + kOffP);
    constexpr uint32_t IDESC_S = idesc_f16(128, 16, 1, 1);         // K tile x queries
    constexpr uint32_t IDESC_O = idesc_f16(128, 16, 1, 1, 1, 0);   // V tile (MN-major) x P
    const uint64_t dK0 = smem_desc(sKV, 16, 1024, 2);
    const uint64_t dV0 = smem_desc(sKV + 2 * kSlab, kSlab, 1024, 2);
    const uint64_t dQ0 = smem_desc(sQ, 16, 1024, 2);
    const uint64_t dP0 = smem_desc(sP, 128, kPSbo, 0);
    auto wait_all = [&](uint64_t* bar, uint32_t par) -> bool {
      const bool ok = __all_sync(0xffffffffu, mbar_wait(bar, par, abort_flag, err, 1u));
      tc_fence_after();
      return ok;
    };
    // scores of tile i into S buffer i % 2 (read by the softmax of tile i-2 before it
    // published P(i-2), which this warp waited for before issuing O(i-2))
    auto issue_s = [&](int i) -> bool {
      const int st = i % kDStages;
      if (!wait_all(&m->full[st], (i / kDStages) & 1)) return false;
      if (leader) {
        const uint64_t dK = dK0 + (uint64_t)((st * kStageBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < kDD / 16; ++kk)
          mma_ss(tmem + (i & 1) * 16, dK + (uint64_t)((kk >> 2) * (kSlab >> 4) + (kk & 3) * 2),
                 dQ0 + (uint64_t)((kk >> 2) * 128 + (kk & 3) * 2), IDESC_S, kk > 0 ? 1u : 0u);
        mma_commit(&m->s_full[i & 1]);
      }
      __syncwarp();
      return true;
    };
    // O(i) = V_i^T P_i^T into O buffer i % 2 (folded by the softmax group before it
    // published P(i-1)); the commit to empty frees the stage once both MMAs have read it
    auto issue_o = [&](int i) -> bool {
      const int st = i % kDStages;
      if (!wait_all(&m->p_ready[i & 1], (i >> 1) & 1)) return false;
      if (leader) {
        const uint64_t dV = dV0 + (uint64_t)((st * kStageBytes) >> 4);
        const uint64_t dP = dP0 + (uint64_t)(((i & 1) * kPBuf) >> 4);
#pragma unroll
        for (int kk = 0; kk < kTok / 16; ++kk)
          mma_ss(tmem + 32 + (i & 1) * 16, dV + (uint64_t)(kk * (2048 >> 4)), dP + (uint64_t)(kk * 16), IDESC_O,
                 kk > 0 ? 1u : 0u);
        mma_commit(&m->o_full[i & 1]);
        mma_commit(&m->empty[st]);
      }
      __syncwarp();
      return true;
    };
    bool ok = wait_all(&m->q_full, 0);
    if (ok) ok = issue_s(0);
    if (ok && nt > 1) ok = issue_s(1);
    for (int i = 0; ok && i < nt; ++i) {
      ok = issue_o(i);
      if (ok && i + 2 < nt) ok = issue_s(i + 2);
    }
    // every MMA issued by this warp completes before TMEM is freed
    if (leader) mma_commit(&m->drain);
    __syncwarp();
    int never = 0;
    mbar_wait(&m->drain, 0, &never, err, 1u);
  } else {
    // ============================================================ softmax (warps 0-3)
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    const int t = warp * 32 + lane;         // token of the tile (scores), dimension (fold)
    float m_run[GQ], l_part[GQ], acc[GQ], al_prev[GQ];
#pragma unroll
    for (int j = 0; j < GQ; ++j) {
      m_run[j] = -INFINITY;
      l_part[j] = 0.f;
      acc[j] = 0.f;
      al_prev[j] = 0.f;
    }
    bool failed = false;
    auto fold = [&](int i, const float (&alpha)[GQ]) {
      // acc = acc * alpha(i) + O(i): both relative to the running max after tile i
      uint32_t v[16];
      tmem_ld16(lane_base + 32 + (i & 1) * 16, v);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < GQ; ++j) acc[j] = fmaf(acc[j], alpha[j], __uint_as_float(v[j]));
    };
    for (int i = 0; i < nt; ++i) {
      // (warp-uniform waits: the tcgen05.ld that follow need converged warps)
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&m->s_full[i & 1], (i >> 1) & 1, abort_flag, err, 1u));
      tc_fence_after();
      uint32_t v[16];
      tmem_ld16(lane_base + (i & 1) * 16, v);
      tmem_wait_ld();
      const bool valid = (long long)i * kTok + t < S;
      float s[GQ];
#pragma unroll
      for (int j = 0; j < GQ; ++j) {
        s[j] = valid ? __uint_as_float(v[j]) * scale_log2 : -INFINITY;
        const float mx = warp_max(s[j]);
        if (lane == 0) m->red[i & 1][warp][j] = mx;
      }
      tc_fence_before();
      if (softmax_sync_or(!ok)) {
        failed = true;
        break;
      }
      float al[GQ];
      // P(i) goes to buffer i % 2, last read by O(i-2), which the fold of tile i-2 waited for
      unsigned char* pt = smem + kOffP + (i & 1) * kPBuf;
#pragma unroll
      for (int j = 0; j < GQ; ++j) {
        const float* r = m->red[i & 1][0] + j;
        const float mc = fmaxf(fmaxf(r[0], r[16]), fmaxf(r[32], r[48]));
        const float mn = fmaxf(m_run[j], mc);
        al[j] = exp2f(m_run[j] - mn);        // 0 while m_run = -inf
        const float p = exp2f(s[j] - mn);
        m_run[j] = mn;
        l_part[j] = fmaf(l_part[j], al[j], p);
        *reinterpret_cast<__nv_bfloat16*>(pt + core_off(j, t, kPSbo)) = __float2bfloat16_rn(p);
      }
      fence_proxy_async_smem();
      named_bar_sync(1, 128);
      if (tid == 0) mbar_arrive(&m->p_ready[i & 1]);
      // fold the previous tile's O (its MMAs ran meanwhile)
      if (i >= 1) {
        const bool ok2 =
            __all_sync(0xffffffffu, mbar_wait(&m->o_full[(i - 1) & 1], ((i - 1) >> 1) & 1, abort_flag, err, 1u));
        tc_fence_after();
        if (ok2) fold(i - 1, al_prev);
        tc_fence_before();
      }
#pragma unroll
      for (int j = 0; j < GQ; ++j) al_prev[j] = al[j];
    }
    if (!failed) {
      const bool ok =
          __all_sync(0xffffffffu, mbar_wait(&m->o_full[(nt - 1) & 1], ((nt - 1) >> 1) & 1, abort_flag, err, 1u));
      tc_fence_after();
      if (ok) fold(nt - 1, al_prev);
      // l_j = sum over the tile threads of their partial sums (all relative to the final max)
#pragma unroll
      for (int j = 0; j < GQ; ++j) {
        const float sum = warp_sum(l_part[j]);
        if (lane == 0) m->red[0][warp][j] = sum;
      }
      failed = softmax_sync_or(!ok || *abort_flag);
      if (!failed) {
        __nv_bfloat16* o = out + (size_t)qrow * kDD + t;
#pragma unroll
        for (int j = 0; j < GQ; ++j) {
          const float* r = m->red[0][0] + j;
          o[(size_t)j * kDD] = __float2bfloat16_rn(acc[j] / ((r[0] + r[16]) + (r[32] + r[48])));
        }
      }
    }
    if (failed) {
      __nv_bfloat16* o = out + (size_t)qrow * kDD + t;
#pragma unroll
      for (int j = 0; j < GQ; ++j) o[(size_t)j * kDD] = __float2bfloat16_rn(__int_as_float(0x7fc00000));
    }
  }

  // ------------------------------------------------------------------ teardown
  __syncwarp();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 dense_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// bf16 tensor map, 128-byte swizzle, boxes of 64 columns x box_rows rows (x 1 unit).
bool dense_map(CUtensorMap* tm, const void* base, int rank, const cuuint64_t* dims, const cuuint64_t* strides,
               uint32_t box_rows) {
  auto enc = dense_encode_fn();
  if (!enc) return false;
  const cuuint32_t box[3] = {64, box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int GQ>
cudaError_t launch_dense_tc(int B, int L, int Hkv, int Hq, long long S, const void* k, const void* v,
                            const void* q, void* out, cudaStream_t s) {
  const unsigned long long units = (unsigned long long)B * L * Hkv;
  CUtensorMap tmK, tmV, tmQ;
  const cuuint64_t kv_dims[3] = {kDD, (cuuint64_t)S, units};
  const cuuint64_t kv_strides[2] = {kDD * 2, (cuuint64_t)S * kDD * 2};
  const cuuint64_t q_dims[2] = {kDD, (cuuint64_t)L * B * Hq};
  const cuuint64_t q_strides[1] = {kDD * 2};
  if (!dense_map(&tmK, k, 3, kv_dims, kv_strides, kTok) || !dense_map(&tmV, v, 3, kv_dims, kv_strides, kTok) ||
      !dense_map(&tmQ, q, 2, q_dims, q_strides, 16))
    return cudaErrorInvalidValue;
  auto kern = dense_tc_kernel<GQ>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kDenseSmem);
  if (e != cudaSuccess) return e;
  kern<<<(unsigned)units, kDThreads, kDenseSmem, s>>>(B, L, Hkv, Hq, S, tmK, tmV, tmQ,
                                                     static_cast<__nv_bfloat16*>(out),
                                                     1.4426950408889634f / sqrtf((float)kDD));
  return cudaGetLastError();
}

// ============================================================== CUDA-core kernel
// One CTA per (sequence, layer, KV head) streams its K and V once, in blocks of 256 tokens:
// thread t scores token t against every query head of the unit (16-byte loads of its key
// row), the block's softmax update is a warp reduction per head, and thread (head, dim pair)
// accumulates P.V with coalesced 4-byte loads of V.

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
      float mx = -INFINITY;
      for (int t = lane; t < nb; t += 32) mx = fmaxf(mx, p[j * kBlock + t]);
      mx = warp_max(mx);
      const float mnew = fmaxf(stat[j], mx);
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
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const bool tc_ok = head_dim == kDD && (reinterpret_cast<uintptr_t>(q) & 15) == 0 && seq_len < (1ll << 31) &&
                     (long long)n_layers * batch * n_q_heads < (1ll << 31) && dense_encode_fn() != nullptr;
  if (tc_ok) {
    cudaError_t e = cudaErrorNotSupported;
    switch (g) {
      case 1: e = launch_dense_tc<1>(batch, n_layers, n_kv_heads, n_q_heads, seq_len, k, v, q, out, s); break;
      case 2: e = launch_dense_tc<2>(batch, n_layers, n_kv_heads, n_q_heads, seq_len, k, v, q, out, s); break;
      case 4: e = launch_dense_tc<4>(batch, n_layers, n_kv_heads, n_q_heads, seq_len, k, v, q, out, s); break;
      case 8: e = launch_dense_tc<8>(batch, n_layers, n_kv_heads, n_q_heads, seq_len, k, v, q, out, s); break;
      case 16: e = launch_dense_tc<16>(batch, n_layers, n_kv_heads, n_q_heads, seq_len, k, v, q, out, s); break;
      default: break;
    }
    if (e != cudaErrorNotSupported) return e == cudaSuccess ? LOWRAM_OK : LOWRAM_ECUDA;
  }
  const size_t smem = sizeof(float) * ((size_t)g * head_dim * 2 + (size_t)g * kBlock + 3 * g);
  cudaError_t e = cudaFuncSetAttribute(dense_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return LOWRAM_ECUDA;
  dense_kernel<<<(unsigned)units, kThreads, smem, s>>>(
      batch, n_layers, n_kv_heads, n_q_heads, head_dim, seq_len, static_cast<const __nv_bfloat16*>(k),
      static_cast<const __nv_bfloat16*>(v), static_cast<const __nv_bfloat16*>(q),
      static_cast<__nv_bfloat16*>(out), 1.4426950408889634f / sqrtf((float)head_dim));
  return cudaGetLastError() == cudaSuccess ? LOWRAM_OK : LOWRAM_ECUDA;
}
