// Reuse of rebuilt chunks across decode steps (rit.work "lowram-kv-cache-compression",
// section "Значения предсказывают, ключи раскладывают по общему базису": each step reuses data
// it has already reconstructed).  A store keeps, per (sequence, layer, KV head, chunk slot),
// the chunk's rebuilt values vhat_t = W2 silu(W1' a_t) + delta_t (bf16, C x d): the part of a
// chunk whose rebuild costs the predictor.  A decode step then splits its selection:
//   reuse_plan_kernel   per unit, hits (chunks the store holds) and misses (the rest)
//   (shard_scan_kernel) the misses as an explicit tile list for the chunk-attention kernel
//   reuse_hit_kernel    per unit, attention over the hits: logits from the coefficient tile
//                       and the projected queries, values from the store (warp MMAs)
//   (combine)           pieces of the misses + the hits' record + the raw tail
//   reuse_fill_kernel   the first fill_cap misses rebuilt into store entries (tcgen05: the
//                       predictor's two layers, then the residual rows added)
//   reuse_commit_kernel the table: first-in first-out entries, evictions, counters.
// Hits are decided against the store as it was before the step; the hit kernel runs before
// the fill kernel overwrites any entry.  Shapes: bf16 native stores, d = 128, h = 256,
// r in {64, 128}, C = 128, g in {4, 8}.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "lowram_internal.cuh"
#include "reuse.cuh"
#include "tc_ptx.cuh"
#include "warp_mma.cuh"

namespace lowram {
namespace {

using namespace tc;

constexpr int kD = 128, kH = 256, kC = 128;

// ------------------------------------------------------------------------------- plan
// One warp per unit: each selected chunk (lane i < k) looked up in the table.  The misses
// replace the unit's selection list (ascending chunk id kept) for the tile-list scan; the
// hits go to the store's per-unit hit list.
__global__ void __launch_bounds__(32)
reuse_plan_kernel(Geom g, Scratch sc, ReuseDev st) {
  const int u = blockIdx.x;
  const Unit un = unit_of(g, u);
  const int l = g.layer0 + un.li;
  const int lane = threadIdx.x;
  const size_t trow = (((size_t)un.b * g.L + l) * g.Hkv + un.hkv) * st.table_stride;
  int n_hit = 0, n_miss = 0;
  for (int i0 = 0; i0 < g.k; i0 += 32) {
    const int i = i0 + lane;
    const bool valid = i < g.k;
    const int slot = valid ? sc.sel_slot[(size_t)u * g.k + i] : 0;
    const int e = valid ? st.table[trow + slot] : -1;
    const bool hit = valid && e >= 0;
    const bool miss = valid && e < 0;
    const unsigned bh = __ballot_sync(0xffffffffu, hit), bm = __ballot_sync(0xffffffffu, miss);
    const unsigned below = (1u << lane) - 1u;
    __syncwarp();   // every lane has read its slot before the list is rewritten in place
    if (hit) {
      const int p = n_hit + __popc(bh & below);
      st.hit_entry[(size_t)u * g.k + p] = e;
      st.hit_slot[(size_t)u * g.k + p] = slot;
    }
    if (miss) sc.sel_slot[(size_t)u * g.k + n_miss + __popc(bm & below)] = slot;
    n_hit += __popc(bh);
    n_miss += __popc(bm);
  }
  if (lane == 0) {
    if (u == 0) st.ring[1] = st.ring[0];   // the commit kernel's view of the ring position
    st.hit_n[u] = n_hit;
    sc.unit_ntile[u] = n_miss;
    atomicAdd(st.counters + 0, (unsigned long long)n_hit);
    atomicAdd(st.counters + 1, (unsigned long long)n_miss);
  }
}

// -------------------------------------------------------------------------------- hits
// Swizzled staging of 128-row blocks (16-byte chunk c of row r at (c & ~7) | ((c ^ r) & 7)),
// as in the selection kernel: conflict-free ldmatrix without padding.
__device__ __forceinline__ uint32_t swz(int r, int c, int row_bytes) {
  return (uint32_t)(r * row_bytes + (((c & 7) ^ (r & 7)) | (c & ~7)) * 16);
}
__device__ __forceinline__ void cp16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}

template <int R, int GQ>
struct HitSmem {
  static constexpr int PAD = R + 8;                       // padded small-operand row
  static constexpr size_t QB = 0;                         // bf16 [16][PAD]: qt hi / lo rows
  static constexpr size_t PB = QB + 16 * PAD * 2;         // bf16 [16][136]: probabilities hi / lo
  static constexpr size_t RED = PB + 16 * 136 * 2;        // float [2][4][GQ]
  static constexpr size_t A = (RED + 2 * 4 * GQ * 4 + 127) / 128 * 128;   // coefficient rows [128][R]
  static constexpr size_t V = A + kC * R * 2;                              // stored values [128][128]
  static constexpr size_t BYTES = V + kC * kD * 2;
};

// One CTA (4 warps) per unit: its hits one after another, an online softmax over them, the
// record of the tail's format (m in log2 units, l, acc [GQ][d]); m = -inf, l = 0 when none.
template <int R, int GQ>
__global__ void __launch_bounds__(128, 3)
reuse_hit_kernel(Geom g, CacheBuffers cb, Scratch sc, ReuseDev st) {
  using SM = HitSmem<R, GQ>;
  constexpr int PAD = SM::PAD;
  extern __shared__ __align__(128) unsigned char smem[];
  __nv_bfloat16* qb = reinterpret_cast<__nv_bfloat16*>(smem + SM::QB);
  __nv_bfloat16* pb = reinterpret_cast<__nv_bfloat16*>(smem + SM::PB);
  float (*red)[4][GQ] = reinterpret_cast<float (*)[4][GQ]>(smem + SM::RED);
  unsigned char* as = smem + SM::A;
  unsigned char* vs = smem + SM::V;
  const int u = blockIdx.x;
  const Unit un = unit_of(g, u);
  const int l = g.layer0 + un.li;
  const int grp = l / g.G;
  const int NG = g.L / g.G;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gq = lane >> 2, cq = (lane & 3) * 2;
  const int n = st.hit_n[u];
  float* rec = st.hit_part + (size_t)u * g.tail_stride;
  float m_run[GQ], l_run[GQ];
#pragma unroll
  for (int j = 0; j < GQ; ++j) {
    m_run[j] = -INFINITY;
    l_run[j] = 0.f;
  }
  float acc[4][4];   // warp w: dimensions 32 w .. 32 w + 31
#pragma unroll
  for (int nt = 0; nt < 4; ++nt)
#pragma unroll
    for (int x = 0; x < 4; ++x) acc[nt][x] = 0.f;
  if (n > 0) {
    // projected queries (already scaled to log2 units) as bf16 hi rows 0..GQ-1 and lo rows
    // GQ..2GQ-1 of the B operand (N = 2 GQ: one n-tile for GQ = 4, two for GQ = 8)
    for (int it = tid; it < 16 * R; it += 128) {
      const int rr = it / R, c = it % R;
      float v = 0.f;
      if (rr < 2 * GQ) v = sc.qt[((size_t)u * GQ + (rr % GQ)) * R + c];
      __nv_bfloat16 hi, lo;
      wm::split_bf16(v, hi, lo);
      qb[rr * PAD + c] = rr < GQ ? hi : (rr < 2 * GQ ? lo : __float2bfloat16_rn(0.f));
    }
    for (int it = tid; it < 16 * 136 / 8; it += 128)
      *reinterpret_cast<uint4*>(pb + it * 8) = make_uint4(0, 0, 0, 0);
  }
  const __nv_bfloat16* coeff = reinterpret_cast<const __nv_bfloat16*>(cb.coeff) +
                               (((size_t)un.b * NG + grp) * g.Hkv + un.hkv) * (size_t)g.nLs * kC * R;
#pragma unroll 1
  for (int i = 0; i < n; ++i) {
    const int slot = st.hit_slot[(size_t)u * g.k + i];
    const int e = st.hit_entry[(size_t)u * g.k + i];
    const __nv_bfloat16* arow = coeff + (size_t)slot * kC * R;
    const __nv_bfloat16* vrow = st.entries + (size_t)e * kC * kD;
    __syncthreads();   // the previous hit's rows are no longer read
    for (int it = tid; it < kC * (R / 8); it += 128) {
      const int r = it / (R / 8), c = it % (R / 8);
      cp16(as + swz(r, c, R * 2), arow + (size_t)r * R + c * 8);
    }
    for (int it = tid; it < kC * (kD / 8); it += 128) {
      const int r = it >> 4, c = it & 15;
      cp16(vs + swz(r, c, kD * 2), vrow + (size_t)r * kD + c * 8);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncthreads();
    // logits of tokens 32 w .. 32 w + 31: A = coefficient rows, B = the qt hi / lo rows
    float lg[2][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
      float c0[4] = {0.f, 0.f, 0.f, 0.f}, c1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < R / 16; ++ks) {
        uint32_t a[4], b[2];
        wm::ldsm_x4(a, as + swz(32 * warp + 16 * mt + (lane & 15), 2 * ks + (lane >> 4), R * 2));
        wm::ldsm_x2(b, qb + (lane & 7) * PAD + ks * 16 + ((lane >> 3) & 1) * 8);
        wm::mma_bf16(c0, a, b);
        if (GQ == 8) {
          wm::ldsm_x2(b, qb + (8 + (lane & 7)) * PAD + ks * 16 + ((lane >> 3) & 1) * 8);
          wm::mma_bf16(c1, a, b);
        }
      }
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        // head cq + (x & 1): GQ = 8: hi in tile 0, lo in tile 1 of the same lane; GQ = 4:
        // hi in columns 0..3 (lanes with cq < 4), lo in columns 4..7 (two lanes over)
        lg[mt][x] = GQ == 8 ? c0[x] + c1[x] : c0[x] + __shfl_xor_sync(0xffffffffu, c0[x], 2);
      }
    }
    // online softmax per head (column), as the selection kernel's tail
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int x = 0; x < 4; ++x) mx[x & 1] = fmaxf(mx[x & 1], lg[mt][x]);
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
      mnew[x] = j < GQ ? fmaxf(m_run[j], fmaxf(fmaxf(red[0][0][j], red[0][1][j]), fmaxf(red[0][2][j], red[0][3][j])))
                       : 0.f;
    }
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        const int j = cq + (x & 1);
        const int t = 32 * warp + 16 * mt + gq + 8 * (x >> 1);
        if (j < GQ) {
          const float pv = exp2f(lg[mt][x] - mnew[x & 1]);
          ps[x & 1] += pv;
          __nv_bfloat16 hi, lo;
          wm::split_bf16(pv, hi, lo);
          pb[j * 136 + t] = hi;
          pb[(GQ + j) * 136 + t] = lo;
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
    float alpha[GQ];
#pragma unroll
    for (int j = 0; j < GQ; ++j) {
      const float mb = fmaxf(fmaxf(red[0][0][j], red[0][1][j]), fmaxf(red[0][2][j], red[0][3][j]));
      const float mn = fmaxf(m_run[j], mb);
      alpha[j] = exp2f(m_run[j] - mn);
      l_run[j] = l_run[j] * alpha[j] + (red[1][0][j] + red[1][1][j]) + (red[1][2][j] + red[1][3][j]);
      m_run[j] = mn;
    }
    float a0 = 0.f, a1 = 0.f;   // the factors of accumulator rows gq and gq + 8 (selected
#pragma unroll                 // without a dynamic index, which would put alpha in memory)
    for (int j = 0; j < GQ; ++j) {
      if (gq < 2 * GQ && gq % GQ == j) a0 = alpha[j];
      if (gq + 8 < 2 * GQ && (gq + 8) % GQ == j) a1 = alpha[j];
    }
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      acc[nt][0] *= a0;
      acc[nt][1] *= a0;
      acc[nt][2] *= a1;
      acc[nt][3] *= a1;
    }
#pragma unroll
    for (int ks = 0; ks < kC / 16; ++ks) {
      uint32_t a[4];
      wm::ldsm_x4(a, pb + (lane & 15) * 136 + ks * 16 + (lane >> 4) * 8);
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        uint32_t b[2];
        wm::ldsm_x2_t(b, vs + swz(ks * 16 + (lane & 15), 4 * warp + nt, kD * 2));
        wm::mma_bf16(acc[nt], a, b);
      }
    }
  }
  // the record: hi and lo rows of head j are accumulator rows j and GQ + j
  if (GQ == 8) {
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      const int dd = 32 * warp + 8 * nt + cq;
      rec[2 * GQ + gq * kD + dd] = acc[nt][0] + acc[nt][2];
      rec[2 * GQ + gq * kD + dd + 1] = acc[nt][1] + acc[nt][3];
    }
  } else {
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      const float o0 = acc[nt][0] + __shfl_xor_sync(0xffffffffu, acc[nt][0], 16);
      const float o1 = acc[nt][1] + __shfl_xor_sync(0xffffffffu, acc[nt][1], 16);
      if (gq < GQ) {
        const int dd = 32 * warp + 8 * nt + cq;
        rec[2 * GQ + gq * kD + dd] = o0;
        rec[2 * GQ + gq * kD + dd + 1] = o1;
      }
    }
  }
#pragma unroll
  for (int j = 0; j < GQ; ++j)
    if (tid == j) {
      rec[j] = m_run[j];
      rec[GQ + j] = l_run[j];
    }
}

// -------------------------------------------------------------------------------- fills
// Persistent CTAs over the first n_fill tiles of the miss list; tile x goes to entry
// (ring + x) mod E.  Per tile, with the chunk's 128 tokens as the MMAs' M dimension:
//   D1^T = A . (W1'/2)^T (SS, M = 128 tokens, N = 128 per hidden half, K = r)
//   H^T  = silu(2 D1^T) as fp16 pairs over the first 128 of the tile's TMEM columns
//   D2^T = H^T . W2^T    (TS: A = H from TMEM, B = W2 in fp16; N = 128 value dims, K = 256)
// then each thread (one token) adds its residual row, if the token has one, and writes its
// 256-byte row of the entry.  Two tiles in flight: tile i of the CTA's range uses TMEM
// columns [256 (i%2), +256) and coefficient stage i%2; warps 0-3 take the even tiles, 4-7
// the odd ones; warp 8 issues the copies and the MMAs.
constexpr int kFillThreads = 288;

template <int R>
struct FillLayout {
  static constexpr int KSLABS = R / 64;
  static constexpr int W1_HALF = KSLABS * 16384;
  static constexpr int W2_BYTES = 4 * 16384;
  static constexpr int A_BYTES = KSLABS * 16384;
  static constexpr int OFF_W1 = 0;
  static constexpr int OFF_W2 = OFF_W1 + 2 * W1_HALF;
  static constexpr int OFF_A = OFF_W2 + W2_BYTES;   // two stages
  static constexpr int OFF_MISC = OFF_A + 2 * A_BYTES;
  static constexpr int SMEM = OFF_MISC + 256 + 1024;
  static_assert(SMEM <= 227 * 1024, "shared memory");
};

struct FillMisc {
  uint64_t w_full, drain, a_full[2], a_empty[2], d1_full[2], h_ready[2], d2_full[2], slot_free[2];
  uint32_t tmem_base;
  int abort_flag;
};

template <int R>
__global__ void __launch_bounds__(kFillThreads, 1)
reuse_fill_kernel(Geom g, CacheBuffers cb, Scratch sc, ReuseDev st, const __grid_constant__ CUtensorMap tmW1,
                  const __grid_constant__ CUtensorMap tmW2, const __grid_constant__ CUtensorMap tmA) {
  using Lay = FillLayout<R>;
  extern __shared__ unsigned char fill_smem_dyn[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(fill_smem_dyn) + 1023) & ~uintptr_t(1023));
  FillMisc* misc = reinterpret_cast<FillMisc*>(smem + Lay::OFF_MISC);
  volatile int* abort_flag = &misc->abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int NG = g.L / g.G;
  const long long n_fill = min((long long)*sc.tile_total, (long long)st.fill_cap);
  const long long x0 = n_fill * blockIdx.x / gridDim.x, x1 = n_fill * (blockIdx.x + 1) / gridDim.x;
  const long long n = x1 - x0;
  const int ring = *st.ring;
  uint32_t* err = sc.err;
  if (tid == 0) {
    mbar_init(&misc->w_full, 1);
    mbar_init(&misc->drain, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&misc->a_full[s], 1);
      mbar_init(&misc->a_empty[s], 1);
      mbar_init(&misc->d1_full[s], 1);
      mbar_init(&misc->h_ready[s], 4);
      mbar_init(&misc->d2_full[s], 1);
      mbar_init(&misc->slot_free[s], 4);
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
    constexpr uint32_t IDESC_1 = idesc_f16(128, 128, 1, 1);   // A (bf16) x W1'/2 (bf16), both K-major
    constexpr uint32_t IDESC_2 = idesc_f16(128, 128, 0, 0);   // H (TMEM, fp16) x W2 (fp16, K-major)
    auto wait_all = [&](uint64_t* bar, uint32_t par) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, par, abort_flag, err, ERR_TIMEOUT));
    };
    auto seg_of = [&](long long i) {
      const Unit un = unit_of(g, sc.tile_unit[x0 + i]);
      return (g.layer0 + un.li) * g.Hkv + un.hkv;
    };
    auto issue_a = [&](long long i) {   // tile i's coefficient tile into stage i % 2
      const int u = sc.tile_unit[x0 + i], slot = sc.tile_slot[x0 + i];
      const Unit un = unit_of(g, u);
      const int grp = (g.layer0 + un.li) / g.G;
      const long long arow = ((((long long)un.b * NG + grp) * g.Hkv + un.hkv) * g.nLs + slot) * kC;
      if (leader) {
        mbar_expect_tx(&misc->a_full[i & 1], (uint32_t)Lay::A_BYTES);
        for (int ks = 0; ks < Lay::KSLABS; ++ks)
          tma_load_2d(smem + Lay::OFF_A + (i & 1) * Lay::A_BYTES + ks * 16384, &tmA, &misc->a_full[i & 1], ks * 64,
                      (int)arow);
      }
      __syncwarp();
    };
    uint32_t ph_w = 0, ph_drain = 0;
    long long a_waited = 0, a_issued = 0;
    bool ok = true, w_pending = false;
    auto load_w = [&](int seg) -> bool {   // W1' halves and W2 of this (layer, KV head)
      w_pending = true;
      if (leader) {
        mbar_expect_tx(&misc->w_full, (uint32_t)(2 * Lay::W1_HALF + Lay::W2_BYTES));
        for (int h2 = 0; h2 < 2; ++h2)
          for (int ks = 0; ks < Lay::KSLABS; ++ks)
            tma_load_2d(smem + Lay::OFF_W1 + h2 * Lay::W1_HALF + ks * 16384, &tmW1, &misc->w_full, ks * 64,
                        seg * kH + h2 * 128);
        for (int j = 0; j < 4; ++j) tma_load_2d(smem + Lay::OFF_W2 + j * 16384, &tmW2, &misc->w_full, j * 64, seg * kD);
      }
      __syncwarp();
      if (!wait_all(&misc->w_full, ph_w)) return false;
      ph_w ^= 1;
      w_pending = false;
      return true;
    };
    auto issue_d1 = [&](long long i) -> bool {
      const int s = (int)(i & 1);
      if (!wait_all(&misc->a_full[s], (uint32_t)((i >> 1) & 1))) return false;
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
    auto drain_mmas = [&](volatile int* flag) -> bool {
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
        const int next_seg = has_next ? seg_of(i + 1) : cur_seg;
        const bool same = has_next && next_seg == cur_seg;
        if (same && !(ok = issue_d1(i + 1))) break;
        if (!(ok = issue_d2(i))) break;
        if (has_next && !same) {
          if (!(ok = drain_mmas(abort_flag))) break;
          cur_seg = next_seg;
          if (!(ok = load_w(cur_seg) && issue_d1(i + 1))) break;
        }
        if (i + 2 < n) {
          if (!(ok = wait_all(&misc->a_empty[i & 1], (uint32_t)((i >> 1) & 1)))) break;
          issue_a(i + 2);
          a_issued = i + 3;
        }
      }
      volatile int never = 0;
      drain_mmas(&never);
      if (!ok && leader) {
        for (long long i = a_waited; i < a_issued; ++i)
          mbar_wait(&misc->a_full[i & 1], (uint32_t)((i >> 1) & 1), &never, err, ERR_TIMEOUT);
        if (w_pending) mbar_wait(&misc->w_full, ph_w, &never, err, ERR_TIMEOUT);
      }
    }
  } else {
    // ============================================================ silu and epilogue
    const int grp_t = warp >> 2;
    const int wq = warp & 3;
    const int t = 32 * wq + lane;                      // this thread's token (TMEM lane)
    const uint32_t lane_off = (uint32_t)(32 * wq) << 16;
    const __nv_bfloat16* rv = reinterpret_cast<const __nv_bfloat16*>(cb.res_val);
    for (long long i = grp_t; i < n; i += 2) {
      const long long x = x0 + i;
      const int s = (int)(i & 1);
      const uint32_t par = (uint32_t)((i >> 1) & 1);
      const int u = sc.tile_unit[x], slot = sc.tile_slot[x];   // (used after the silu)
      if (!__all_sync(0xffffffffu, mbar_wait(&misc->d1_full[s], par, abort_flag, err, ERR_TIMEOUT))) break;
      tc_fence_after();
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
      // while the second GEMM runs: this token's residual record, if it has one (the chunk's
      // few records scanned), and its row
      const Unit un = unit_of(g, u);
      const int l = g.layer0 + un.li;
      const int32_t* rptr = cb.res_ptr + (((size_t)un.b * g.L + l) * g.Hkv + un.hkv) * (g.nLs + 1);
      int r0 = rptr[slot], r1 = rptr[slot + 1];
      if (r0 < 0 || r1 < r0 || (long long)r1 > (long long)cb.n_records) {
        if (t == 0) atomicOr(err, ERR_RES_PTR);
        r0 = r1 = 0;
      }
      int rec = -1;
      for (int k = r0; k < r1; ++k)
        if ((int)cb.res_pos[k] == t) rec = k;
      uint4 drow[kD / 8];
      const uint4* dp = reinterpret_cast<const uint4*>(rv + (size_t)(rec < 0 ? 0 : rec) * kD);
#pragma unroll
      for (int j = 0; j < kD / 8; ++j) drow[j] = rec >= 0 ? __ldg(dp + j) : make_uint4(0, 0, 0, 0);
      if (!__all_sync(0xffffffffu, mbar_wait(&misc->d2_full[s], par, abort_flag, err, ERR_TIMEOUT))) break;
      tc_fence_after();
      // vhat[t] = D2[t] + delta (if the token has a record), as bf16, straight to the entry,
      // 64 dims per TMEM round trip
      uint4* dst = reinterpret_cast<uint4*>(st.entries + ((size_t)((ring + x) % st.E) * kC + t) * kD);
#pragma unroll
      for (int hv = 0; hv < 2; ++hv) {
        uint32_t vd[64];
        tmem_ld32(tmem + lane_off + 256 * s + 128 + 64 * hv, *reinterpret_cast<uint32_t(*)[32]>(vd));
        tmem_ld32(tmem + lane_off + 256 * s + 128 + 64 * hv + 32, *reinterpret_cast<uint32_t(*)[32]>(vd + 32));
        tmem_wait_ld();
        if (hv == 1) {   // the tile's TMEM is free for its slot's next tile
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&misc->slot_free[s]);
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint4 dr = drow[8 * hv + j];
          const uint32_t dw[4] = {dr.x, dr.y, dr.z, dr.w};
          uint32_t o[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float a = __uint_as_float(vd[8 * j + 2 * k]) + __uint_as_float(dw[k] << 16);
            const float b = __uint_as_float(vd[8 * j + 2 * k + 1]) + __uint_as_float(dw[k] & 0xffff0000u);
            const __nv_bfloat162 p = __floats2bfloat162_rn(a, b);
            o[k] = *reinterpret_cast<const uint32_t*>(&p);
          }
          dst[8 * hv + j] = make_uint4(o[0], o[1], o[2], o[3]);
        }
      }
    }
  }
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------------------ commit
// The table after the fills: entry (ring + x) mod E now holds tile x of the miss list; its
// previous chunk leaves the table.  Then the ring and the fill counter advance.  One thread
// per fill: the call's fills have distinct chunks and distinct entries, and no chunk they
// evict is one of them (an evicted chunk was in the table, so it was a hit, not a miss).
// The ring position comes from ring[1] (copied by the plan kernel), so the thread that
// advances ring[0] races with no reader.
__global__ void __launch_bounds__(256)
reuse_commit_kernel(Geom g, Scratch sc, ReuseDev st) {
  const long long n_fill = min((long long)*sc.tile_total, (long long)st.fill_cap);
  const int ring = st.ring[1];
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    st.ring[0] = (int)((ring + n_fill) % st.E);
    st.counters[2] += (unsigned long long)n_fill;
  }
  for (long long x = (long long)blockIdx.x * blockDim.x + threadIdx.x; x < n_fill; x += (long long)gridDim.x * blockDim.x) {
    const int u = sc.tile_unit[x], slot = sc.tile_slot[x];
    const Unit un = unit_of(g, u);
    const int l = g.layer0 + un.li;
    const long long key = (((long long)un.b * g.L + l) * g.Hkv + un.hkv) * st.table_stride + slot;
    const int e = (int)((ring + x) % st.E);
    const long long old = st.owner[e];
    if (old >= 0 && st.table[old] == e) st.table[old] = -1;
    st.owner[e] = key;
    st.table[key] = e;
  }
}

PFN_cuTensorMapEncodeTiled_v12000 map_encoder() {
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

// 2-D 16-bit map over [rows][inner], boxes of 64 x box_rows in the 128-byte swizzle layout.
bool map16(CUtensorMap* m, const void* base, bool f16, uint64_t inner, uint64_t rows, uint32_t box_rows) {
  auto enc = map_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base),
             dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int R, int GQ>
cudaError_t run_reuse(const Geom& g, const CacheBuffers& cb, const Scratch& sc, const ReuseDev& st, const void* w1f_tc,
                      int n_sm, cudaStream_t s, int phase) {
  cudaError_t e;
  if (phase == 0) {   // plan + tile list
    reuse_plan_kernel<<<g.U, 32, 0, s>>>(g, sc, st);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    return launch_tile_scan(g, sc, s);
  }
  if (phase == 1) {   // hits
    using SM = HitSmem<R, GQ>;
    auto k = reuse_hit_kernel<R, GQ>;
    if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SM::BYTES)) != cudaSuccess) return e;
    k<<<g.U, 128, SM::BYTES, s>>>(g, cb, sc, st);
    return cudaGetLastError();
  }
  // fills + commit
  using Lay = FillLayout<R>;
  CUtensorMap tmW1, tmW2, tmA;
  const uint64_t lh = (uint64_t)g.L * g.Hkv;
  const uint64_t rows = (uint64_t)g.B * (g.L / g.G) * g.Hkv * g.nLs * kC;
  if (!map16(&tmW1, w1f_tc, false, R, lh * kH, 128) || !map16(&tmW2, st.w2h, true, kH, lh * kD, 128) ||
      !map16(&tmA, cb.coeff, false, R, rows, kC))
    return cudaErrorInvalidValue;
  auto k = reuse_fill_kernel<R>;
  if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::SMEM)) != cudaSuccess) return e;
  k<<<n_sm, kFillThreads, Lay::SMEM, s>>>(g, cb, sc, st, tmW1, tmW2, tmA);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  reuse_commit_kernel<<<(unsigned)std::min<long long>(((long long)g.U * g.k + 255) / 256, 4LL * n_sm), 256, 0, s>>>(g, sc, st);
  return cudaGetLastError();
}

}  // namespace

bool reuse_supported(const Geom& g, int dtype, int store) {
  return dtype == LOWRAM_BF16 && store == LOWRAM_STORE_NATIVE && g.d == kD && g.h == kH && g.C == kC &&
         (g.r == 64 || g.r == 128) && (g.g == 4 || g.g == 8) && map_encoder() != nullptr;
}

cudaError_t launch_reuse(const Geom& g, const CacheBuffers& cb, const Scratch& sc, const ReuseDev& st,
                         const void* w1f_tc, int n_sm, cudaStream_t s, int phase) {
  if (g.r == 128 && g.g == 4) return run_reuse<128, 4>(g, cb, sc, st, w1f_tc, n_sm, s, phase);
  if (g.r == 128 && g.g == 8) return run_reuse<128, 8>(g, cb, sc, st, w1f_tc, n_sm, s, phase);
  if (g.r == 64 && g.g == 4) return run_reuse<64, 4>(g, cb, sc, st, w1f_tc, n_sm, s, phase);
  if (g.r == 64 && g.g == 8) return run_reuse<64, 8>(g, cb, sc, st, w1f_tc, n_sm, s, phase);
  return cudaErrorNotSupported;
}

}  // namespace lowram
