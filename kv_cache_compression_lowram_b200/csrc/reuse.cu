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

// ------------------------------------------------------------------------------- fills
// Persistent CTAs over the first n_fill tiles of the miss list; tile x goes to entry
// (ring + x) mod E.  Per tile, like the encoder's predictor pass: the coefficient tile by TMA,
// D1_hh = (W1'_hh / 2) A^T (SS, M = 128 hidden rows, N = C tokens), H = silu(2 D1) as fp16 in
// shared memory (MN-major), D2 = W2 H (SS, M = 128 value dims, N = C), then vhat = D2 plus the
// chunk's residual rows, assembled as bf16 [C][d] in shared memory and written to the entry
// by one bulk copy.  Latency hiding within the CTA: the residual rows are staged by cp.async
// while the MMAs run; the next tile's coefficient tile (and W1', W2 at a new (layer, KV head))
// are requested as soon as the current tile's MMAs are done, i.e. during its epilogue; the
// next tile's unit, slot and record range are read one tile ahead.
constexpr int kFillResStage = 32;   // residual rows of a chunk staged in shared memory

template <int R>
struct FillLayout {
  static constexpr int KSLABS = R / 64;
  static constexpr int W1_HALF = KSLABS * 16384;
  static constexpr int W2_BYTES = 4 * 16384;
  static constexpr int H_HALF = 2 * 16384;                   // 128 hidden rows x 128 tokens, fp16
  static constexpr int A_BYTES = KSLABS * 16384;
  static constexpr int OFF_W1 = 0;
  static constexpr int OFF_W2 = OFF_W1 + 2 * W1_HALF;
  static constexpr int OFF_AH = OFF_W2 + W2_BYTES;           // the A tile, then H half 0
  static constexpr int OFF_H1 = OFF_AH + (A_BYTES > H_HALF ? A_BYTES : H_HALF);   // H half 1, then vhat
  static constexpr int OFF_RES = OFF_H1 + H_HALF;            // bf16 [kFillResStage][d]
  static constexpr int OFF_MISC = OFF_RES + kFillResStage * kD * 2;
  static constexpr int SMEM = OFF_MISC + 64 + kC * 4 + 1024;
  static_assert(kC * kD * 2 <= H_HALF, "vhat tile fits the H half-1 buffer");
  static_assert(SMEM <= 227 * 1024, "shared memory");
};

template <int R>
__global__ void __launch_bounds__(256, 1)
reuse_fill_kernel(Geom g, CacheBuffers cb, Scratch sc, ReuseDev st, const __grid_constant__ CUtensorMap tmW1,
                  const __grid_constant__ CUtensorMap tmW2, const __grid_constant__ CUtensorMap tmA) {
  using Lay = FillLayout<R>;
  extern __shared__ unsigned char fill_smem_dyn[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(fill_smem_dyn) + 1023) & ~uintptr_t(1023));
  uint64_t* bar_w = reinterpret_cast<uint64_t*>(smem + Lay::OFF_MISC);
  uint64_t* bar_in = bar_w + 1;
  uint64_t* bar_mma = bar_w + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_w + 3);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* tok_rec = reinterpret_cast<int*>(smem + Lay::OFF_MISC + 64);   // [C]: token -> record, or -1
  const __nv_bfloat16* res_s = reinterpret_cast<const __nv_bfloat16*>(smem + Lay::OFF_RES);
  __nv_bfloat16* out_s = reinterpret_cast<__nv_bfloat16*>(smem + Lay::OFF_H1);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int NG = g.L / g.G;
  const long long n_fill = min((long long)*sc.tile_total, (long long)st.fill_cap);
  const long long x0 = n_fill * blockIdx.x / gridDim.x, x1 = n_fill * (blockIdx.x + 1) / gridDim.x;
  const int ring = *st.ring;
  uint32_t* err = sc.err;
  const __nv_bfloat16* rv = reinterpret_cast<const __nv_bfloat16*>(cb.res_val);
  if (tid == 0) {
    mbar_init(bar_w, 1);
    mbar_init(bar_in, 1);
    mbar_init(bar_mma, 1);
    *abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
  const uint64_t dW1 = smem_desc(smem_u32(smem + Lay::OFF_W1), 16, 1024, 2);
  const uint64_t dW2 = smem_desc(smem_u32(smem + Lay::OFF_W2), 16, 1024, 2);
  const uint64_t dA = smem_desc(smem_u32(smem + Lay::OFF_AH), 16, 1024, 2);
  const uint64_t dH0 = smem_desc(smem_u32(smem + Lay::OFF_AH), 16384, 1024, 2);   // MN-major
  const uint64_t dH1 = smem_desc(smem_u32(smem + Lay::OFF_H1), 16384, 1024, 2);
  constexpr uint32_t IDESC_1 = idesc_f16(128, kC, 1, 1);         // W1'/2 (bf16) x A (bf16)
  constexpr uint32_t IDESC_2 = idesc_f16(128, kC, 0, 0, 0, 1);   // W2 (f16) x H (f16, MN-major)
  uint32_t ph_w = 0, ph_in = 0, ph_mma = 0;
  bool w_pending = false, a_pending = false;   // copies requested and not yet waited for
  bool m_pending = false;                      // MMAs committed and not yet waited for
  int cur_seg = -1;
  bool ok = true;
  const int hh = warp >> 2;                 // silu: hidden half; epilogue: token half
  const int row = 32 * (warp & 3) + lane;   // TMEM lane: hidden unit in the half / value dim

  // tile x's unit, slot, (layer, KV head) and record range
  struct TileRef {
    int u, slot, seg, r0, r1;
    long long arow;
  };
  auto tile_ref = [&](long long x) {
    TileRef t;
    t.u = sc.tile_unit[x];
    t.slot = sc.tile_slot[x];
    const Unit un = unit_of(g, t.u);
    const int l = g.layer0 + un.li, grp = l / g.G;
    t.seg = l * g.Hkv + un.hkv;
    t.arow = ((((long long)un.b * NG + grp) * g.Hkv + un.hkv) * g.nLs + t.slot) * kC;
    const int32_t* rptr = cb.res_ptr + (((size_t)un.b * g.L + l) * g.Hkv + un.hkv) * (g.nLs + 1);
    t.r0 = rptr[t.slot];
    t.r1 = rptr[t.slot + 1];
    return t;
  };
  // tid 0, once no MMA reads the buffers: the copies of tile t (W1', W2 only at a new pair)
  auto issue_loads = [&](const TileRef& t, int seg_now) {
    if (t.seg != seg_now) {
      mbar_expect_tx(bar_w, (uint32_t)(2 * Lay::W1_HALF + Lay::W2_BYTES));
      for (int h2 = 0; h2 < 2; ++h2)
        for (int ks = 0; ks < Lay::KSLABS; ++ks)
          tma_load_2d(smem + Lay::OFF_W1 + h2 * Lay::W1_HALF + ks * 16384, &tmW1, bar_w, ks * 64, t.seg * kH + h2 * 128);
      for (int j = 0; j < 4; ++j) tma_load_2d(smem + Lay::OFF_W2 + j * 16384, &tmW2, bar_w, j * 64, t.seg * kD);
    }
    mbar_expect_tx(bar_in, (uint32_t)(Lay::KSLABS * kC * 128));
    for (int ks = 0; ks < Lay::KSLABS; ++ks)
      tma_load_2d(smem + Lay::OFF_AH + ks * 16384, &tmA, bar_in, ks * 64, (int)t.arow);
  };

  TileRef cur{};
  if (x0 < x1) {
    cur = tile_ref(x0);
    if (tid == 0) issue_loads(cur, -1);
  }
  for (long long x = x0; ok && x < x1; ++x) {
    // this tile's copies were issued (before the loop, or during the last tile's epilogue)
    const bool new_seg = cur.seg != cur_seg;
    w_pending = w_pending || new_seg;
    a_pending = true;
    cur_seg = cur.seg;
    int r0 = cur.r0, r1 = cur.r1;
    if (r0 < 0 || r1 < r0 || (long long)r1 > (long long)cb.n_records) {
      if (tid == 0) atomicOr(err, ERR_RES_PTR);
      r0 = r1 = 0;
    }
    // residual rows r0 .. r0 + 31 into shared memory (cp.async), and the token -> record map
    const int nst = min(r1 - r0, kFillResStage);
    for (int i = tid; i < nst * (kD / 8); i += 256) {
      const int rr = i / (kD / 8), c = i % (kD / 8);
      cp16(smem + Lay::OFF_RES + (rr * kD + c * 8) * 2, rv + (size_t)(r0 + rr) * kD + c * 8);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
    for (int t = tid; t < kC; t += 256) tok_rec[t] = -1;   // filled once the MMAs are issued
    // (a phase flips only once every thread has passed its wait, so that the drain below
    // waits for the phase a failed wait was on)
    if (new_seg) {
      ok = mbar_wait(bar_w, ph_w, abort_flag, err, ERR_TIMEOUT);
      if (!__syncthreads_and(ok)) break;
      ph_w ^= 1;
      w_pending = false;
    }
    ok = mbar_wait(bar_in, ph_in, abort_flag, err, ERR_TIMEOUT);
    if (!__syncthreads_and(ok)) break;
    ph_in ^= 1;
    a_pending = false;
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2)
#pragma unroll
        for (int kk = 0; kk < R / 16; ++kk) {
          const uint64_t ko = (uint64_t)((kk >> 2) * 1024 + (kk & 3) * 2);
          mma_ss(tmem + h2 * kC, dW1 + (uint64_t)((h2 * Lay::W1_HALF) >> 4) + ko, dA + ko, IDESC_1, kk > 0 ? 1u : 0u);
        }
      mma_commit(bar_mma);
      bulk_wait_read_all();   // the last tile's vhat (in the H half-1 buffer) has been copied out
    }
    // while the pre-activations run: the token -> record map (the barrier above ordered the
    // reset) and the next tile's reference (both dependent global loads)
    for (int i = r0 + tid; i < r1; i += 256) {
      const int pos = cb.res_pos[i];
      if (pos < kC) tok_rec[pos] = i;
    }
    TileRef nxt{};
    if (x + 1 < x1) nxt = tile_ref(x + 1);
    m_pending = true;
    ok = mbar_wait(bar_mma, ph_mma, abort_flag, err, ERR_TIMEOUT);
    if (!__syncthreads_and(ok)) break;
    ph_mma ^= 1;
    m_pending = false;
    tc_fence_after();
    {   // silu -> H_hh (fp16) in shared memory, MN-major: hidden row `row`, 8 tokens per 16 bytes
      unsigned char* hrow = smem + (hh == 0 ? Lay::OFF_AH : Lay::OFF_H1) + (row >> 3) * 1024 + (row & 7) * 128;
#pragma unroll
      for (int q = 0; q < kC / 32; ++q) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_off + hh * kC + q * 32, v);
        tmem_wait_ld();
        uint32_t hv[16];
#pragma unroll
        for (int j = 0; j < 16; ++j)
          hv[j] = silu_half2_of_halfx(pack_f16x2(__uint_as_float(v[2 * j]), __uint_as_float(v[2 * j + 1])));
        unsigned char* blk = hrow + (q >> 1) * 16384;
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
          const int c16 = (q & 1) * 4 + k4;
          *reinterpret_cast<uint4*>(blk + ((c16 ^ (row & 7)) << 4)) =
              make_uint4(hv[4 * k4], hv[4 * k4 + 1], hv[4 * k4 + 2], hv[4 * k4 + 3]);
        }
      }
    }
    tc_fence_before();
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {   // D2 = W2 . H over both hidden halves
      tc_fence_after();
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2)
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const int slab = h2 * 2 + (kk >> 2);
          mma_ss(tmem + 2 * kC, dW2 + (uint64_t)((slab * 16384 + (kk & 3) * 32) >> 4),
                 (h2 == 0 ? dH0 : dH1) + (uint64_t)((kk * 2048) >> 4), IDESC_2, (h2 | kk) ? 1u : 0u);
        }
      mma_commit(bar_mma);
    }
    m_pending = true;
    ok = mbar_wait(bar_mma, ph_mma, abort_flag, err, ERR_TIMEOUT);
    asm volatile("cp.async.wait_group 0;" ::: "memory");   // this thread's residual rows
    if (!__syncthreads_and(ok)) break;
    ph_mma ^= 1;
    m_pending = false;
    tc_fence_after();
    // every MMA of this tile is done: the next tile's copies go out now
    if (tid == 0 && x + 1 < x1) issue_loads(nxt, cur_seg);
    // vhat[t][row] = D2[row][t] + delta_t[row] for tokens hh * 64 .. + 63, into shared memory
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      uint32_t v[32];
      tmem_ld32(tmem + lane_off + 2 * kC + hh * 64 + q * 32, v);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int t = hh * 64 + q * 32 + j;
        float val = __uint_as_float(v[j]);
        const int ri = tok_rec[t];   // the same for the whole warp
        if (ri >= 0) {
          const int si = ri - r0;
          val += __bfloat162float(si < kFillResStage ? res_s[si * kD + row] : rv[(size_t)ri * kD + row]);
        }
        out_s[t * kD + row] = __float2bfloat16_rn(val);
      }
    }
    tc_fence_before();
    fence_proxy_async_smem();
    __syncthreads();   // vhat complete; tok_rec and the staged rows are free again
    if (tid == 0) {
      bulk_store(st.entries + (size_t)((ring + x) % st.E) * kC * kD, out_s, (uint32_t)(kC * kD * 2));
      bulk_commit();
    }
    cur = nxt;
  }
  if (tid == 0) {
    bulk_wait_all();
    if (!ok) {   // a wait gave up: let the copies this CTA started land before it exits
      volatile int never = 0;
      if (w_pending) mbar_wait(bar_w, ph_w, &never, err, ERR_TIMEOUT);
      if (a_pending) mbar_wait(bar_in, ph_in, &never, err, ERR_TIMEOUT);
      if (m_pending) mbar_wait(bar_mma, ph_mma, &never, err, ERR_TIMEOUT);   // TMEM is freed below
    }
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  __syncthreads();
  if (warp == 0) {
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
  k<<<n_sm, 256, Lay::SMEM, s>>>(g, cb, sc, st, tmW1, tmW2, tmA);
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
