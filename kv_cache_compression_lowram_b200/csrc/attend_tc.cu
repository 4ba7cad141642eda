// Steps 3-5 on tcgen05 tensor cores (sm_100a): rebuild the selected chunks on chip and
// attend over them, fused in one persistent kernel.
//
// Per selected chunk of C tokens (coefficient rows A_c, C x r, bf16; fp16 when the cache
// stores int8 rows, see below) of a unit:
//   S  = A_c . Qt^T                 scores q_j . khat_t / sqrt(d) * log2(e) in the low-rank
//                                   form (Qt_j = B_l q_j, "OjaKV" 3.1 projects queries into
//                                   the key basis); M=128 tokens, N=16 heads (g used)
//   D1 = W1'_hh/2 . A_c^T           pre-activations / 2 of the predictor's hidden layer,
//                                   W1' = W1 B_l^T (exact fold of W1 khat_t); a sub-tile is
//                                   one half hh of the 256 hidden units: M=128 hidden rows,
//                                   N=C tokens, both operands in shared memory
//   H  = silu(2 * D1) = u + u tanh(u), written back to TMEM as fp16 (MUFU tanh)
//   D3 = H . P                      softmax-weighted hidden sums per head (A = H from TMEM,
//                                   B = P, the chunk's probabilities, fp16 in SMEM)
//   D4 = Delta^T . P_res            softmax-weighted residual rows delta_t of the flagged
//                                   tokens (A = the rows as TMA loads them, MN-major; B = the
//                                   probabilities at those tokens, bf16 / fp16)
// while a softmax warpgroup keeps the online max/sum per head.  The predictor's second
// layer is applied once per unit in the combine kernel: sum_t p_t (W2 h_t + delta_t) =
// W2 (sum_t p_t h_t) + sum_t p_t delta_t.  Key rebuild: "LowRAM Compresses KV Cache
// Asymmetrically", section "Cross-Layer Low-Rank Key Compression"; values: same page,
// "Core Mechanism" (Vhat = f(K), delta kept for the worst tokens); attention: "OjaKV", 3.
//
// Warp roles (16 warps): 0 TMA producer (tiles, queries, residual rows, W1' halves), 1 MMA
// issuer + TMEM owner, 2-3 int8 converters (idle for a native store), 4-7 and 8-11 the silu
// epilogue groups of hidden halves 0 and 1, 12-15 softmax, the P / P_res tiles and the
// accumulation of the chunks' D3 / D4.
// A warp reaches TMEM lanes 32*(warp%4) .. +31, so each warpgroup of four consecutive
// warps covers all 128 lanes.
// Sub-tile n (hidden half n % 2 of chunk n / 2) has D1 buffer n % 3: with three buffers for
// two epilogue groups the pre-activations of sub-tile n+3 are computed while the epilogue
// still works on n+1 and n+2, so neither the tensor core nor the epilogue waits for the
// other's round trip.  W1' lives in shared memory (the SS form costs no more tensor time at
// N=128 than the TS form, and frees the 128 TMEM columns the third buffer needs).
// TMEM (512 columns): D1 buffers [0,384), S double buffer [384,416), D3 double buffer x 2
// halves [416,480), D4 double buffer [480,512).
// Every wait is bounded: on timeout the kernel raises the error word, drains its own
// copies and MMAs, frees TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "lowram_internal.cuh"
#include "tc_ptx.cuh"

namespace lowram {
namespace {

using namespace tc;

constexpr int kThreadsTC = 512;   // 16 warps: register allocation rounds to whole warpgroups
constexpr int kEpiWarp0 = 4;      // first hidden-row epilogue warp
constexpr int kSoftWarp0 = 12;    // first softmax warp
constexpr int kHid = 256;
constexpr int kDh = 128;
constexpr int kResCap = kResPad;  // residual records per chunk handled by the tensor cores
static_assert(kResCap == 32, "the P_res tile and the D4 MMAs assume 32 records");

// I8: the cache stores coefficients and residual rows as int8 with an fp16 scale per row
// ("LowRAM Compresses KV Cache Asymmetrically", composition with quantisation); they arrive
// in an int8 staging ring and warps 2-3 write the scaled tiles as fp16 (every integer of
// |x| <= 127 and its product with the scale fit fp16 with 11 significant bits, and the
// conversion needs no int-to-float instructions, which share a unit with the epilogue's
// tanh).  The operands that meet them in an MMA (W1', the projected queries, P_res) are fp16
// too.
template <int R, int C, bool I8>
struct TcLayout {
  static constexpr int SUBS = 2;                     // sub-tiles per chunk = hidden halves
  static constexpr int NBUF = 3;                     // D1 buffers
  static constexpr int STAGES = I8 ? 2 : 3;
  static constexpr int KSLABS = R / 64;
  static constexpr int A_STAGE = KSLABS * 16384;     // 128 rows x 128 B per 64-wide K slab
  static constexpr int W_HALF = KSLABS * 16384;      // 128 hidden rows x R of W1'/2, same layout
  static constexpr int Q_BUF = KSLABS * 2048;        // 16 rows x 128 B per slab
  static constexpr int P_BUF = 16 * C * 2;
  static constexpr int P_SBO = (C / 8) * 128;
  static constexpr int RES_SLAB = kResCap * 128;     // 32 records x 64 dims (128 B)
  static constexpr int RES_BUF = 2 * RES_SLAB;
  static constexpr int PR_BUF = 16 * kResCap * 2;
  static constexpr int PR_SBO = (kResCap / 8) * 128;
  static constexpr int OFF_W = 0;
  static constexpr int OFF_A = OFF_W + 2 * W_HALF;
  static constexpr int OFF_Q = OFF_A + STAGES * A_STAGE;
  static constexpr int OFF_RES = OFF_Q + 2 * Q_BUF;
  static constexpr int OFF_P = OFF_RES + STAGES * RES_BUF;
  static constexpr int OFF_PR = OFF_P + 2 * P_BUF;
  static constexpr int SA_SLOT = C * R + C * 2;           // int8 tile + fp16 row scales
  static constexpr int SR_SLOT = kResCap * kDh;            // int8 residual rows
  static constexpr int OFF_SA = OFF_PR + 2 * PR_BUF;
  static constexpr int OFF_SR = OFF_SA + (I8 ? 2 * SA_SLOT : 0);
  static constexpr int OFF_MISC = OFF_SR + (I8 ? 2 * SR_SLOT : 0);
  static constexpr int MISC_BYTES = 3072;
  static constexpr int SMEM = OFF_MISC + MISC_BYTES + 1024;   // + alignment slack
  // TMEM columns
  static constexpr uint32_t T_D1 = 0;
  static constexpr uint32_t T_S = 384;
  static constexpr uint32_t T_D3 = 416;
  static constexpr uint32_t T_D4 = 480;
  static constexpr uint32_t TMEM_COLS = 512;
  static_assert(SMEM <= 227 * 1024, "shared memory budget");
  static_assert(SA_SLOT % 16 == 0 && OFF_SA % 16 == 0, "bulk copies need 16-byte alignment");
  static_assert(OFF_A % 1024 == 0 && OFF_Q % 1024 == 0 && OFF_RES % 1024 == 0,
                "128-byte-swizzled operands need 1024-byte alignment");
};

struct Bars {
  uint64_t a_full[4], a_empty[4];     // coefficient tiles
  uint64_t r_full[4], r_empty[4];     // residual rows (+ their record range and token map)
  uint64_t q_full[2], q_empty[2];
  uint64_t s_full[2];
  uint64_t d1_full[3], h_ready[3];   // per D1 buffer
  uint64_t p_ready[2];
  uint64_t d3_full[2];
  uint64_t stg_full[2], stg_empty[2];   // int8 coefficient staging (int8 store)
  uint64_t rstg_full[2], rstg_empty[2]; // int8 residual staging (int8 store)
  uint64_t w1_ready;   // W1' of the next (layer, KV head) is in shared memory
  uint64_t seg_done;   // every MMA that read the previous W1' is complete
  uint64_t drain;
  uint64_t h_free[3];  // the weighted sums of the H in a D1 buffer are complete (bf16 split issue)
  uint64_t drain2;
};

struct Misc {
  Bars bars;
  int stage_rec[4][2];               // residual record range [r0, r1) of the chunk in a stage
  int8_t stage_idx[4][128];          // token -> its record index if below kResCap, else -1
  __half stage_rs[4][32];            // int8 store: scales of the first kResCap records (0 past)
  float red_max[4][16];
  float red_sum[4][16];
  uint32_t tmem_base;
  int abort_flag;
};

static_assert(sizeof(Misc) <= 3072, "Misc must fit its shared-memory slot");

// Sequential walk over a CTA's chunk tiles: the unit of each chunk, the chunk's index in its
// unit and the unit's (layer, KV head) segment, updated by counters (no division per step).
struct TileWalk {
  int ci, u, rem, seg, ub, k, B;
  __device__ __forceinline__ void init(long long x0, int k_, int B_) {
    k = k_;
    B = B_;
    ci = 0;
    u = (int)(x0 / k);
    rem = (int)(x0 - (long long)u * k);
    seg = u / B;
    ub = u - seg * B;
  }
  __device__ __forceinline__ void advance_to(int target) {
    while (ci < target) {
      ++ci;
      if (++rem == k) {
        rem = 0;
        ++u;
        if (++ub == B) {
          ub = 0;
          ++seg;
        }
      }
    }
  }
  __device__ __forceinline__ bool next_starts_segment() const { return rem + 1 == k && ub + 1 == B; }
  __device__ __forceinline__ bool first_of_unit() const { return rem == 0; }
};

// The same walk over an explicit tile list (context-sharded decode: a unit holds any number
// of the call's tiles, 0 .. k): tile x belongs to unit tu[x].  The next tile's unit is read
// one step ahead, so its latency hides under the current tile's work.
struct TileWalkList {
  const int32_t* tu;
  long long x0, x1;
  int ci, u, seg, B, nu;
  bool first;
  __device__ __forceinline__ void init(long long x0_, long long x1_, const int32_t* tu_, int B_) {
    tu = tu_;
    x0 = x0_;
    x1 = x1_;
    B = B_;
    ci = 0;
    u = x0 < x1 ? __ldg(tu + x0) : 0;
    first = x0 == 0 || (x0 < x1 && __ldg(tu + x0 - 1) != u);
    seg = u / B;
    nu = x0 + 1 < x1 ? __ldg(tu + x0 + 1) : -1;
  }
  __device__ __forceinline__ void advance_to(int target) {
    while (ci < target) {
      ++ci;
      first = nu != u;
      u = nu;
      seg = u / B;
      nu = x0 + ci + 1 < x1 ? __ldg(tu + x0 + ci + 1) : -1;
    }
  }
  // only asked while a next tile exists in this CTA's range
  __device__ __forceinline__ bool next_starts_segment() const { return nu / B != seg; }
  __device__ __forceinline__ bool first_of_unit() const { return first; }
};
template <bool CT> struct WalkOf { using type = TileWalk; };
template <> struct WalkOf<true> { using type = TileWalkList; };

// Offset of element (row j, column k) in a K-major operand tile without swizzle: 8 x 16-byte
// core matrices, K-adjacent ones 128 bytes apart, 8-row groups sbo bytes apart.
__device__ __forceinline__ uint32_t kmajor_off(int j, int k, int sbo) {
  return (uint32_t)((j >> 3) * sbo + (k >> 3) * 128 + (j & 7) * 16 + (k & 7) * 2);
}

// One 16-bit MMA operand element: fp16 for the int8 variant, bf16 otherwise.
template <bool F16>
__device__ __forceinline__ void st_op16(unsigned char* p, float v) {
  if (F16)
    *reinterpret_cast<__half*>(p) = __float2half_rn(v);
  else
    *reinterpret_cast<__nv_bfloat16*>(p) = __float2bfloat16_rn(v);
}

// Four int8 values (one 32-bit word, lowest byte first) times a scale, as two fp16 pairs.
// Flipping the sign bit gives x + 128 as an unsigned byte u; the fp16 with bit pattern
// 0x6400 | u is 1024 + u exactly, so subtracting 1152 gives x exactly, and the product with
// the scale is rounded once (to nearest).
__device__ __forceinline__ void i8x4_scaled_f16(uint32_t w, __half2 scale, uint32_t& lo, uint32_t& hi) {
  const uint32_t u = w ^ 0x80808080u;
  const uint32_t m01 = __byte_perm(u, 0x64646464u, 0x4140);   // (1024 + u0, 1024 + u1)
  const uint32_t m23 = __byte_perm(u, 0x64646464u, 0x4342);   // (1024 + u2, 1024 + u3)
  const __half2 bias = __halves2half2(__ushort_as_half((unsigned short)0x6480), __ushort_as_half((unsigned short)0x6480));
  const __half2 x01 = __hmul2(__hsub2(*reinterpret_cast<const __half2*>(&m01), bias), scale);
  const __half2 x23 = __hmul2(__hsub2(*reinterpret_cast<const __half2*>(&m23), bias), scale);
  lo = *reinterpret_cast<const uint32_t*>(&x01);
  hi = *reinterpret_cast<const uint32_t*>(&x23);
}

// TW: the main-loop waits take the call's limit (the test hook that exercises the abort path);
// otherwise every wait has the compile-time default and compiles to the plain bounded wait.
// CT: the tiles come as an explicit list (sc.tile_unit / sc.tile_slot, sc.tile_total of them)
// instead of k per unit.
template <int R, int C, int GQ, bool I8, bool TW, bool CT>
__global__ void __launch_bounds__(kThreadsTC, 1)
attend_tc_kernel(Geom g, CacheBuffers cb, Scratch sc, const __grid_constant__ CUtensorMap tmW,
                 const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmQ,
                 const __grid_constant__ CUtensorMap tmRes) {
  using Lay = TcLayout<R, C, I8>;
  constexpr int SUBS = Lay::SUBS, STAGES = Lay::STAGES, KSLABS = Lay::KSLABS, NBUF = Lay::NBUF;
  extern __shared__ unsigned char smem_dyn[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
  Misc* misc = reinterpret_cast<Misc*>(smem + Lay::OFF_MISC);
  Bars& bar = misc->bars;
  volatile int* abort_flag = &misc->abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  using Walk = typename WalkOf<CT>::type;
  const long long total = CT ? (long long)*sc.tile_total : (long long)g.U * g.k;
  const int32_t* tslot = CT ? sc.tile_slot : sc.sel_slot;   // storage slot of tile x
  const long long x0 = tile_begin(total, g.P, blockIdx.x);
  const long long x1 = tile_begin(total, g.P, blockIdx.x + 1);
  const int NCH = (int)(x1 - x0);
  const int NS = NCH * SUBS;
  const int NG = g.L / g.G;
  uint32_t* err = sc.err;
  // limit of the main-loop waits (the drain waits at an abort keep the full kWaitCycles)
  const long long wlim = TW ? g.wait_cycles : kWaitCycles;
  auto init_walk = [&](Walk& w, long long a, long long b) {
    if constexpr (CT) w.init(a, b, sc.tile_unit, g.B);
    else w.init(a, g.k, g.B);
  };

  // ------------------------------------------------------------------ set-up
  if (tid == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&bar.a_full[i], I8 ? 2 : 1);   // the two converter warps, or the TMA arrive
      mbar_init(&bar.a_empty[i], 1);
      mbar_init(&bar.r_full[i], I8 ? 2 : 1);
      mbar_init(&bar.r_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar.stg_full[i], 1);
      mbar_init(&bar.stg_empty[i], 2);
      mbar_init(&bar.rstg_full[i], 1);
      mbar_init(&bar.rstg_empty[i], 2);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar.q_full[i], 1);
      mbar_init(&bar.q_empty[i], 1);
      mbar_init(&bar.s_full[i], 1);
      mbar_init(&bar.p_ready[i], 1);
      mbar_init(&bar.d3_full[i], 1);
    }
    for (int i = 0; i < NBUF; ++i) {
      mbar_init(&bar.d1_full[i], 1);
      mbar_init(&bar.h_ready[i], 4);      // the 4 warps of the sub-tile's epilogue group
      mbar_init(&bar.h_free[i], 1);
    }
    mbar_init(&bar.drain2, 1);
    mbar_init(&bar.w1_ready, 1);          // TMA
    mbar_init(&bar.seg_done, 1);
    mbar_init(&bar.drain, 1);
    misc->abort_flag = 0;
    mbar_init_fence();
  }
  // zero the P and P_res tiles (rows >= g stay zero for the whole kernel)
  for (int i = tid; i < (2 * Lay::P_BUF + 2 * Lay::PR_BUF) / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(smem + Lay::OFF_P)[i] = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
  if (warp == 1) {
    tmem_alloc(&misc->tmem_base, Lay::TMEM_COLS);
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc->tmem_base;
  // the set-up above overlaps the selection kernel's end (programmatic dependent launch);
  // its outputs (projected queries, selected slots) are read only from here on
  grid_dep_launch();
  grid_dep_wait();

  const uint32_t sW = smem_u32(smem + Lay::OFF_W);
  const uint32_t sA = smem_u32(smem + Lay::OFF_A);
  const uint32_t sQ = smem_u32(smem + Lay::OFF_Q);
  const uint32_t sP = smem_u32(smem + Lay::OFF_P);
  const uint32_t sRes = smem_u32(smem + Lay::OFF_RES);
  const uint32_t sPR = smem_u32(smem + Lay::OFF_PR);
  constexpr int F16B = I8 ? 0 : 1;   // operand format of the tile MMAs: 1 = bf16, 0 = fp16
  constexpr uint32_t IDESC_S = idesc_f16(128, 16, F16B, F16B);        // tile x queries
  constexpr uint32_t IDESC_1 = idesc_f16(128, C, F16B, F16B);         // W1' half x tile
  constexpr uint32_t IDESC_3 = idesc_f16(128, 16, 0, 0);              // H (TMEM, fp16) x P (fp16)
  constexpr uint32_t IDESC_4 = idesc_f16(128, 16, F16B, F16B, 1, 0);  // residual rows (MN-major) x P_res

  if (warp == 0) {
    // ============================================================ TMA producer
    // The whole warp walks the tiles (waits and bookkeeping are warp-uniform); one elected
    // lane issues the copies.
    const bool leader = elect_one();
    if (NCH > 0) {
      int unit_i = -1, prev_u = -1, issued_a = 0, issued_r = 0, q_issued = 0;
      int seg_i = -1, prev_seg = -1, w1_issued = 0;
      Walk wk;
      init_walk(wk, x0, x1);
      for (int ci = 0; ci < NCH; ++ci) {
        const long long x = x0 + ci;
        wk.advance_to(ci);
        const int u = wk.u;
        if (u != prev_u) {
          ++unit_i;
          prev_u = u;
          const int qb = unit_i & 1;
          if (unit_i >= 2 && !__all_sync(0xffffffffu, mbar_wait(&bar.q_empty[qb], ((unit_i >> 1) - 1) & 1,
                                                                abort_flag, err, ERR_TIMEOUT, wlim)))
            break;
          if (leader) {
            mbar_expect_tx(&bar.q_full[qb], 16 * R * 2);
#pragma unroll
            for (int ks = 0; ks < KSLABS; ++ks)
              tma_load_2d(smem + Lay::OFF_Q + qb * Lay::Q_BUF + ks * 2048, &tmQ, &bar.q_full[qb], ks * 64, u * 16);
          }
          __syncwarp();
          q_issued = unit_i + 1;
        }
        const int st = ci % STAGES, s2 = ci & 1;
        const uint32_t par = ((ci / STAGES) - 1) & 1;
        if (I8) {   // the int8 tile goes to the staging ring; the converters fill stage st
          if (ci >= 2 && !__all_sync(0xffffffffu, mbar_wait(&bar.stg_empty[s2], ((ci >> 1) - 1) & 1, abort_flag,
                                                            err, ERR_TIMEOUT, wlim)))
            break;
        } else if (ci >= STAGES &&
                   !__all_sync(0xffffffffu, mbar_wait(&bar.a_empty[st], par, abort_flag, err, ERR_TIMEOUT, wlim))) {
          break;
        }
        const Unit un = unit_of(g, u);
        const int l = g.layer0 + un.li;
        const int grp = l / g.G;
        const int slot = tslot[x];
        const int row0 = (int)(((((long long)un.b * NG + grp) * g.Hkv + un.hkv) * g.nLs + slot) * C);
        if (leader) {
          if (I8) {
            unsigned char* dst = smem + Lay::OFF_SA + s2 * Lay::SA_SLOT;
            mbar_expect_tx(&bar.stg_full[s2], (uint32_t)Lay::SA_SLOT);
            bulk_load(dst, static_cast<const unsigned char*>(cb.coeff) + (size_t)row0 * R, (uint32_t)(C * R),
                      &bar.stg_full[s2]);
            bulk_load(dst + C * R, cb.coeff_scale + row0, (uint32_t)(C * 2), &bar.stg_full[s2]);
          } else {
            mbar_expect_tx(&bar.a_full[st], (uint32_t)(C * R * 2));
#pragma unroll
            for (int ks = 0; ks < KSLABS; ++ks)
              tma_load_2d(smem + Lay::OFF_A + st * Lay::A_STAGE + ks * 16384, &tmA, &bar.a_full[st], ks * 64, row0);
          }
        }
        __syncwarp();
        issued_a = ci + 1;
        if (wk.seg != prev_seg) {
          // the first chunk of a (layer, KV head): its W1' halves, once every MMA that read
          // the previous pair's has completed
          ++seg_i;
          prev_seg = wk.seg;
          if (seg_i > 0 && !__all_sync(0xffffffffu, mbar_wait(&bar.seg_done, (seg_i - 1) & 1, abort_flag, err,
                                                              ERR_TIMEOUT, wlim)))
            break;
          if (leader) {
            mbar_expect_tx(&bar.w1_ready, (uint32_t)(2 * Lay::W_HALF));
            const int wrow = (l * g.Hkv + un.hkv) * kHid;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh)
#pragma unroll
              for (int ks = 0; ks < KSLABS; ++ks)
                tma_load_2d(smem + Lay::OFF_W + hh * Lay::W_HALF + ks * 16384, &tmW, &bar.w1_ready, ks * 64,
                            wrow + hh * 128);
          }
          __syncwarp();
          w1_issued = seg_i + 1;
        }
        const int32_t* rptr = cb.res_ptr + (((size_t)un.b * g.L + l) * g.Hkv + un.hkv) * (g.nLs + 1);
        int r0 = rptr[slot], r1 = rptr[slot + 1];
        if (r0 < 0 || r1 < r0 || (long long)r1 > cb.n_records) {   // corrupt CSR offsets: clamp, report
          if (lane == 0) atomicOr(err, ERR_RES_PTR);
          r0 = (int)max(0ll, min((long long)r0, (long long)cb.n_records));
          r1 = (int)max((long long)r0, min((long long)r1, (long long)cb.n_records));
        }
        const int nres = min(r1 - r0, kResCap);
        const int my_pos = lane < nres ? (int)cb.res_pos[r0 + lane] : C;
        const __half my_rs = (I8 && lane < nres) ? cb.res_scale[r0 + lane] : __ushort_as_half((unsigned short)0);
        if (ci >= STAGES && !__all_sync(0xffffffffu, mbar_wait(&bar.r_empty[st], par, abort_flag, err, ERR_TIMEOUT, wlim)))
          break;
        if (I8 && ci >= 2 &&
            !__all_sync(0xffffffffu, mbar_wait(&bar.rstg_empty[s2], ((ci >> 1) - 1) & 1, abort_flag, err, ERR_TIMEOUT, wlim)))
          break;
        if (I8) misc->stage_rs[st][lane] = my_rs;
        // record range and token -> record map for the softmax warps (published by the
        // arrive below); a position outside the chunk is left out of the map
        if (lane == 0) {
          misc->stage_rec[st][0] = r0;
          misc->stage_rec[st][1] = r1;
        }
        for (int w4 = lane; w4 < C / 4; w4 += 32) reinterpret_cast<uint32_t*>(misc->stage_idx[st])[w4] = 0xffffffffu;
        __syncwarp();
        if (my_pos < C) misc->stage_idx[st][my_pos] = (int8_t)lane;
        __syncwarp();
        if (leader) {
          // records r0 .. r0+31 (rows past the chunk's own records meet zero probabilities,
          // and the cache keeps 32 zero rows after its last record): two 64-dim slabs by
          // TMA, or 32 int8 rows into the staging ring
          if (I8) {
            mbar_expect_tx(&bar.rstg_full[s2], (uint32_t)Lay::SR_SLOT);
            bulk_load(smem + Lay::OFF_SR + s2 * Lay::SR_SLOT,
                      static_cast<const unsigned char*>(cb.res_val) + (size_t)r0 * kDh, (uint32_t)Lay::SR_SLOT,
                      &bar.rstg_full[s2]);
          } else {
            mbar_expect_tx(&bar.r_full[st], (uint32_t)Lay::RES_BUF);
            tma_load_2d(smem + Lay::OFF_RES + st * Lay::RES_BUF, &tmRes, &bar.r_full[st], 0, r0);
            tma_load_2d(smem + Lay::OFF_RES + st * Lay::RES_BUF + Lay::RES_SLAB, &tmRes, &bar.r_full[st], 64, r0);
          }
        }
        __syncwarp();
        issued_r = ci + 1;
      }
      if (*abort_flag && leader) {
        // let every copy this warp started land before the CTA's shared memory goes away
        volatile int never = 0;
        if (I8) {
          for (int ci = max(0, issued_a - 2); ci < issued_a; ++ci)
            mbar_wait(&bar.stg_full[ci & 1], (ci >> 1) & 1, &never, err, ERR_TIMEOUT);
          for (int ci = max(0, issued_r - 2); ci < issued_r; ++ci)
            mbar_wait(&bar.rstg_full[ci & 1], (ci >> 1) & 1, &never, err, ERR_TIMEOUT);
        } else {
          for (int ci = max(0, issued_a - STAGES); ci < issued_a; ++ci)
            mbar_wait(&bar.a_full[ci % STAGES], (ci / STAGES) & 1, &never, err, ERR_TIMEOUT);
          for (int ci = max(0, issued_r - STAGES); ci < issued_r; ++ci)
            mbar_wait(&bar.r_full[ci % STAGES], (ci / STAGES) & 1, &never, err, ERR_TIMEOUT);
        }
        for (int ui = max(0, q_issued - 2); ui < q_issued; ++ui)
          mbar_wait(&bar.q_full[ui & 1], (ui >> 1) & 1, &never, err, ERR_TIMEOUT);
        if (w1_issued > 0) mbar_wait(&bar.w1_ready, (w1_issued - 1) & 1, &never, err, ERR_TIMEOUT);
      }
    }
  } else if (warp == 1) {
    // ============================================================ MMA issuer
    // The whole warp runs the schedule and waits; one elected lane issues every MMA and
    // commit, so descriptors and TMEM addresses stay warp-uniform.
    const bool leader = elect_one();
    if (NS > 0) {
      int m_unit_i = -1, m_cur_u = -1, m_seg_i = -1, m_cur_seg = -1;
      // Descriptors are built once; a K step, stage, buffer or sub-tile only moves the
      // start address, i.e. adds (byte offset >> 4) to the low field (no carry: every
      // shared address here is below 256 KiB).
      const uint64_t dW0 = smem_desc(sW, 16, 1024, 2);              // W1' halves
      const uint64_t dA0 = smem_desc(sA, 16, 1024, 2);              // coefficient tiles
      const uint64_t dQ0 = smem_desc(sQ, 16, 1024, 2);              // projected queries
      const uint64_t dP0 = smem_desc(sP, 128, Lay::P_SBO, 0);       // probabilities
      const uint64_t dR0 = smem_desc(sRes, Lay::RES_SLAB, 1024, 2); // residual rows, MN-major
      const uint64_t dPR0 = smem_desc(sPR, 128, Lay::PR_SBO, 0);    // probabilities at records
      const uint32_t t_d1 = tmem + Lay::T_D1;
      const uint32_t t_s = tmem + Lay::T_S, t_d3 = tmem + Lay::T_D3, t_d4 = tmem + Lay::T_D4;
      Walk wk;
      init_walk(wk, x0, x1);
      auto wait_all = [&](uint64_t* b, uint32_t par) -> bool {
        return __all_sync(0xffffffffu, mbar_wait(b, par, abort_flag, err, ERR_TIMEOUT, wlim));
      };
      // Pre-activations of sub-tile n (hidden half hh = n % 2 of chunk n / 2) into D1 buffer
      // n % 3; hidden half 0 also carries the chunk's scores (two accumulation chains
      // interleaved).  Tiles, queries and W1' arrive by TMA (or as the converters'
      // proxy-fenced stores): the waits on their barriers order them for the MMAs.  The TMEM
      // this call overwrites was released before barriers the caller has waited and fenced:
      // D1 buffer n % 3 by the epilogue (H of sub-tile n-3, read by the D3 MMAs issued just
      // before), the S buffer of chunk ci by the softmax for chunk ci-2, before it published
      // that chunk's probabilities.
      auto issue_mma1 = [&](int n) -> bool {
        const int ci = n >> 1, hh = n & 1;
        wk.advance_to(ci);
        const int st = ci % STAGES;
        if (hh == 0) {
          if (!wait_all(&bar.a_full[st], (ci / STAGES) & 1)) return false;
          const int u = wk.u;
          if (u != m_cur_u) {
            if (m_cur_u >= 0 && leader) mma_commit(&bar.q_empty[m_unit_i & 1]);
            ++m_unit_i;
            m_cur_u = u;
            if (!wait_all(&bar.q_full[m_unit_i & 1], (m_unit_i >> 1) & 1)) return false;
            const int seg = wk.seg;
            if (seg != m_cur_seg) {
              ++m_seg_i;
              m_cur_seg = seg;
              if (!wait_all(&bar.w1_ready, m_seg_i & 1)) return false;
            }
          }
        }
        const int bf = n % NBUF;
        const uint32_t td = t_d1 + bf * 128;
        const uint64_t dA = dA0 + (uint64_t)((st * Lay::A_STAGE) >> 4);
        const uint64_t dW = dW0 + (uint64_t)((hh * Lay::W_HALF) >> 4);
        if (leader) {
          if (hh == 0) {
            const int sb = ci & 1;
            const uint64_t dQ = dQ0 + (uint64_t)(((m_unit_i & 1) * Lay::Q_BUF) >> 4);
#pragma unroll
            for (int kk = 0; kk < R / 16; ++kk) {
              const uint64_t ko = (uint64_t)((kk >> 2) * 1024 + (kk & 3) * 2);
              const uint32_t acc = kk > 0 ? 1u : 0u;
              mma_ss(t_s + sb * 16, dA + ko, dQ + (uint64_t)((kk >> 2) * 128 + (kk & 3) * 2), IDESC_S, acc);
              mma_ss(td, dW + ko, dA + ko, IDESC_1, acc);
            }
            mma_commit(&bar.s_full[sb]);
            mma_commit(&bar.d1_full[bf]);
          } else {
#pragma unroll
            for (int kk = 0; kk < R / 16; ++kk) {
              const uint64_t ko = (uint64_t)((kk >> 2) * 1024 + (kk & 3) * 2);
              mma_ss(td, dW + ko, dA + ko, IDESC_1, kk > 0 ? 1u : 0u);
            }
            mma_commit(&bar.d1_full[bf]);
            mma_commit(&bar.a_empty[st]);
            if (n + 1 < NS && wk.next_starts_segment())
              mma_commit(&bar.seg_done);   // the last MMA that reads this W1' has been issued
          }
        }
        __syncwarp();
        return true;
      };

      bool ok = true;
      if (!I8) {
        // bf16 store: this warp issues only the pre-activations and the scores, as far ahead
        // as the D1 buffers allow; warp 2 issues the weighted sums as the silu groups finish.
        // D1 buffer n % 3 is reused once the weighted sums of sub-tile n-3 are complete; the
        // scores of chunk ci overwrite those of chunk ci-2 once the softmax has published
        // that chunk's probabilities.
        for (int n = 0; ok && n < NS; ++n) {
          const int ci = n >> 1;
          if (n >= NBUF) ok = wait_all(&bar.h_free[n % NBUF], ((n / NBUF) - 1) & 1);
          if (ok && (n & 1) == 0 && ci >= 2) ok = wait_all(&bar.p_ready[ci & 1], ((ci - 2) >> 1) & 1);
          if (ok) {
            tc_fence_after();
            ok = issue_mma1(n);
          }
        }
      } else {
        for (int n = 0; ok && n < NBUF && n < NS; ++n) ok = issue_mma1(n);
        // Per chunk: the weighted sums of both hidden halves (and the residual rows) back to
        // back, their commit, and only then the next pre-activations.  A commit waits for
        // every MMA this thread issued before it, so D1 work queued between the two halves
        // would hold back the softmax's fold of the chunk, and with it the probabilities of
        // the next chunk.
        for (int ci = 0; ok && ci < NCH; ++ci) {
          const int pb = ci & 1, st = ci % STAGES;
          const uint64_t dP = dP0 + (uint64_t)((pb * Lay::P_BUF) >> 4);
  #pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int n = 2 * ci + hh, bf = n % NBUF;
            if (!wait_all(&bar.h_ready[bf], (n / NBUF) & 1)) { ok = false; break; }
            // One acquire covers the softmax's hand-offs: before it publishes the
            // probabilities of chunk ci it has waited for the chunk's residual rows and read
            // out the D3 / D4 buffer of chunk ci-2.
            if (hh == 0 && !wait_all(&bar.p_ready[pb], (ci >> 1) & 1)) { ok = false; break; }
            tc_fence_after();
            if (leader) {
              // softmax-weighted hidden sums of this half: H (fp16 pairs, token pair j at
              // column j of the buffer) times P, K = the chunk's tokens
  #pragma unroll
              for (int kk = 0; kk < C / 16; ++kk)
                mma_ts(t_d3 + pb * 32 + hh * 16, t_d1 + bf * 128 + kk * 8, dP + (uint64_t)(kk * 16), IDESC_3,
                       kk > 0 ? 1u : 0u);
              if (hh == 0) {
                // the chunk's weighted residual rows: 16 records = two 8-row groups of the
                // MN-major tile per MMA
                const uint64_t dPR = dPR0 + (uint64_t)((pb * Lay::PR_BUF) >> 4);
                const uint64_t dR = dR0 + (uint64_t)((st * Lay::RES_BUF) >> 4);
  #pragma unroll
                for (int kk = 0; kk < kResCap / 16; ++kk)
                  mma_ss(t_d4 + pb * 16, dR + (uint64_t)(kk * (2048 >> 4)), dPR + (uint64_t)(kk * 16), IDESC_4,
                         kk > 0 ? 1u : 0u);
                mma_commit(&bar.r_empty[st]);
              } else {
                mma_commit(&bar.d3_full[pb]);
              }
            }
            __syncwarp();
          }
          // the next pre-activations into the two buffers just read
          for (int n = 2 * ci + NBUF; ok && n < 2 * ci + NBUF + 2 && n < NS; ++n) ok = issue_mma1(n);
        }
      }
      // every MMA this warp issued must finish before TMEM is released
      if (leader) {
        mma_commit(&bar.drain);
        volatile int never = 0;
        mbar_wait(&bar.drain, 0, &never, err, ERR_TIMEOUT);
      }
      __syncwarp();
    }
  } else if (!I8 && warp == 2) {
    // ============================================================ weighted-sum issuer (bf16)
    // Per chunk: the weighted hidden sums of each half as soon as its silu group has written
    // H (and, for half 0, the softmax its probabilities), the residual rows' sum with half
    // 0; a commit per half frees its D1 buffer for the pre-activation warp, and the commit
    // after half 1 hands the chunk to the softmax.  Issued apart from the pre-activations,
    // so waiting for an epilogue group never holds back the next D1 MMAs.
    const bool leader = elect_one();
    if (NS > 0) {
      const uint64_t dP0 = smem_desc(sP, 128, Lay::P_SBO, 0);       // probabilities
      const uint64_t dR0 = smem_desc(sRes, Lay::RES_SLAB, 1024, 2); // residual rows, MN-major
      const uint64_t dPR0 = smem_desc(sPR, 128, Lay::PR_SBO, 0);    // probabilities at records
      const uint32_t t_d1 = tmem + Lay::T_D1, t_d3 = tmem + Lay::T_D3, t_d4 = tmem + Lay::T_D4;
      auto wait_all = [&](uint64_t* b, uint32_t par) -> bool {
        return __all_sync(0xffffffffu, mbar_wait(b, par, abort_flag, err, ERR_TIMEOUT, wlim));
      };
      bool ok = true;
      for (int ci = 0; ok && ci < NCH; ++ci) {
        const int pb = ci & 1, st = ci % STAGES;
        const uint64_t dP = dP0 + (uint64_t)((pb * Lay::P_BUF) >> 4);
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int n = 2 * ci + hh, bf = n % NBUF;
          if (!wait_all(&bar.h_ready[bf], (n / NBUF) & 1)) { ok = false; break; }
          if (hh == 0 && !wait_all(&bar.p_ready[pb], (ci >> 1) & 1)) { ok = false; break; }
          tc_fence_after();
          if (leader) {
#pragma unroll
            for (int kk = 0; kk < C / 16; ++kk)
              mma_ts(t_d3 + pb * 32 + hh * 16, t_d1 + bf * 128 + kk * 8, dP + (uint64_t)(kk * 16), IDESC_3,
                     kk > 0 ? 1u : 0u);
            if (hh == 0) {
              const uint64_t dPR = dPR0 + (uint64_t)((pb * Lay::PR_BUF) >> 4);
              const uint64_t dR = dR0 + (uint64_t)((st * Lay::RES_BUF) >> 4);
#pragma unroll
              for (int kk = 0; kk < kResCap / 16; ++kk)
                mma_ss(t_d4 + pb * 16, dR + (uint64_t)(kk * (2048 >> 4)), dPR + (uint64_t)(kk * 16), IDESC_4,
                       kk > 0 ? 1u : 0u);
              mma_commit(&bar.r_empty[st]);
            }
            mma_commit(&bar.h_free[bf]);
            if (hh == 1) mma_commit(&bar.d3_full[pb]);
          }
          __syncwarp();
        }
      }
      // every MMA this warp issued must finish before TMEM is released
      if (leader) {
        mma_commit(&bar.drain2);
        volatile int never = 0;
        mbar_wait(&bar.drain2, 0, &never, err, ERR_TIMEOUT);
      }
      __syncwarp();
    }
  } else if (I8 && (warp == 2 || warp == 3)) {
    // ============================================================ int8 converters
    // Per chunk: the staged int8 coefficient rows times their fp16 scales become the fp16
    // tile of stage st in the 128-byte-swizzle K-major layout the MMAs read (16-byte piece
    // j of row t at j ^ (t % 8) inside its 64-column slab), and the staged int8 residual
    // rows times their scales become the fp16 MN-major tile of the D4 MMA (same swizzle,
    // rows = records, 64-dim slabs).
    const int ct = tid - 64;   // 0..63
    bool ok = true;
    for (int ci = 0; ok && ci < NCH; ++ci) {
      const int st = ci % STAGES, s2 = ci & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&bar.stg_full[s2], (ci >> 1) & 1, abort_flag, err, ERR_TIMEOUT, wlim));
      if (ok && ci >= STAGES)
        ok = __all_sync(0xffffffffu, mbar_wait(&bar.a_empty[st], ((ci / STAGES) - 1) & 1, abort_flag, err, ERR_TIMEOUT, wlim));
      if (!ok) break;
      {
        const unsigned char* src = smem + Lay::OFF_SA + s2 * Lay::SA_SLOT;
        const __half* scl = reinterpret_cast<const __half*>(src + C * R);
        unsigned char* dst = smem + Lay::OFF_A + st * Lay::A_STAGE;
        constexpr int P16 = R / 16;   // 16-element pieces per row
        for (int it = ct; it < C * P16; it += 64) {
          const int t = it / P16, c16 = it % P16;
          const uint4 q = *reinterpret_cast<const uint4*>(src + t * R + c16 * 16);
          const __half2 sg = __half2half2(scl[t]);
          uint32_t o[8];
          i8x4_scaled_f16(q.x, sg, o[0], o[1]);
          i8x4_scaled_f16(q.y, sg, o[2], o[3]);
          i8x4_scaled_f16(q.z, sg, o[4], o[5]);
          i8x4_scaled_f16(q.w, sg, o[6], o[7]);
          const int col = c16 * 16, ks = col >> 6, j = (col & 63) >> 3;
          unsigned char* row = dst + ks * 16384 + t * 128;
          *reinterpret_cast<uint4*>(row + ((j ^ (t & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
          *reinterpret_cast<uint4*>(row + (((j + 1) ^ (t & 7)) << 4)) = make_uint4(o[4], o[5], o[6], o[7]);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bar.stg_empty[s2]);
        mbar_arrive(&bar.a_full[st]);
      }
      ok = __all_sync(0xffffffffu, mbar_wait(&bar.rstg_full[s2], (ci >> 1) & 1, abort_flag, err, ERR_TIMEOUT, wlim));
      if (ok && ci >= STAGES)
        ok = __all_sync(0xffffffffu, mbar_wait(&bar.r_empty[st], ((ci / STAGES) - 1) & 1, abort_flag, err, ERR_TIMEOUT, wlim));
      if (!ok) break;
      {
        const unsigned char* src = smem + Lay::OFF_SR + s2 * Lay::SR_SLOT;
        unsigned char* dst = smem + Lay::OFF_RES + st * Lay::RES_BUF;
        for (int it = ct; it < kResCap * (kDh / 16); it += 64) {
          const int i = it / (kDh / 16), c16 = it % (kDh / 16);
          const uint4 q = *reinterpret_cast<const uint4*>(src + i * kDh + c16 * 16);
          const __half2 sg = __half2half2(misc->stage_rs[st][i]);
          uint32_t o[8];
          i8x4_scaled_f16(q.x, sg, o[0], o[1]);
          i8x4_scaled_f16(q.y, sg, o[2], o[3]);
          i8x4_scaled_f16(q.z, sg, o[4], o[5]);
          i8x4_scaled_f16(q.w, sg, o[6], o[7]);
          const int dim = c16 * 16, slab = dim >> 6, j = (dim & 63) >> 3;
          unsigned char* row = dst + slab * Lay::RES_SLAB + i * 128;
          *reinterpret_cast<uint4*>(row + ((j ^ (i & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
          *reinterpret_cast<uint4*>(row + (((j + 1) ^ (i & 7)) << 4)) = make_uint4(o[4], o[5], o[6], o[7]);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bar.rstg_empty[s2]);
        mbar_arrive(&bar.r_full[st]);
      }
    }
  } else if (warp >= kEpiWarp0 && warp < kEpiWarp0 + 8) {
    // ============================================================ silu epilogue
    // Warpgroup A (warps 4-7) takes hidden half 0 of every chunk, B (8-11) half 1, all C
    // tokens each, so one group's MUFU work overlaps the other's TMEM round trips.
    const int grp_ab = (warp - kEpiWarp0) >> 2;  // hidden half of this group
    const int wl = warp & 3;
    const uint32_t lane_off = (uint32_t)(wl * 32) << 16;
    for (int n = grp_ab; n < NS; n += 2) {
      const int bf = n % NBUF;
      if (!__all_sync(0xffffffffu, mbar_wait(&bar.d1_full[bf], (n / NBUF) & 1, abort_flag, err, ERR_TIMEOUT, wlim)))
        break;
      tc_fence_after();
      // 64 tokens at a time: their fp32 pre-activations (64 columns) in, their H (fp16
      // pairs, 32 columns) out over the first half of the columns already read, so H of
      // token pair (2j, 2j+1) lands in column j of the buffer
      const uint32_t dcol = tmem + lane_off + Lay::T_D1 + bf * 128;
#pragma unroll
      for (int q = 0; q < C / 64; ++q) {
        uint32_t h[32];
        {
          uint32_t v[32];
          tmem_ld32(dcol + q * 64, v);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 16; ++c)
            h[c] = silu_half2_of_halfx(pack_f16x2(__uint_as_float(v[2 * c]), __uint_as_float(v[2 * c + 1])));
          tmem_ld32(dcol + q * 64 + 32, v);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 16; ++c)
            h[16 + c] = silu_half2_of_halfx(pack_f16x2(__uint_as_float(v[2 * c]), __uint_as_float(v[2 * c + 1])));
        }
        tmem_st32(dcol + q * 32, h);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar.h_ready[bf]);
    }
  } else if (warp >= kSoftWarp0) {
    // ============================================================ softmax + accumulation
    // Per chunk: online max/sum per head, the fp16 P tile and the P_res tile (the
    // probabilities at the flagged tokens) for the MMAs, residual records beyond the first
    // 32 on CUDA cores, and (one chunk later) the chunk's D3 / D4 folded into the running
    // sums.  Thread t is token t for the scores, hidden row t of both halves for D3 and
    // head-dim element t for D4 and the extra records.
    const int w = warp & 3;
    const int t = w * 32 + lane;
    const uint32_t lane_off = (uint32_t)(w * 32) << 16;
    float m_run[GQ], l_run[GQ], accD[GQ], accD4[GQ], accH0[GQ], accH1[GQ], al_prev[GQ];
#pragma unroll
    for (int j = 0; j < GQ; ++j) {
      m_run[j] = -INFINITY; l_run[j] = 0.f; accD[j] = 0.f; accD4[j] = 0.f; accH0[j] = 0.f;
      accH1[j] = 0.f; al_prev[j] = 1.f;
    }
    unsigned char* pbase = smem + Lay::OFF_P;
    unsigned char* prbase = smem + Lay::OFF_PR;
    int cur_u = -1;
    // After a failed wait a warp stops working ("live" false) but keeps passing the named
    // barriers of every remaining chunk, so the other warps of the group never block on it;
    // once the abort flag is up every wait returns at once.
    bool live = true;
    // fold D3 / D4 of chunk c (sums relative to the running max after c) into the totals
    auto fold = [&](int c) {
      const int pb = c & 1;
      live = __all_sync(0xffffffffu, live && mbar_wait(&bar.d3_full[pb], (c >> 1) & 1, abort_flag, err, ERR_TIMEOUT, wlim));
      if (!live) return;
      tc_fence_after();
      uint32_t v0[16], v1[16], v4[16];
      tmem_ld16(tmem + lane_off + Lay::T_D3 + pb * 32, v0);
      tmem_ld16(tmem + lane_off + Lay::T_D3 + pb * 32 + 16, v1);
      tmem_ld16(tmem + lane_off + Lay::T_D4 + pb * 16, v4);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
#pragma unroll
      for (int j = 0; j < GQ; ++j) {
        accH0[j] = fmaf(accH0[j], al_prev[j], __uint_as_float(v0[j]));
        accH1[j] = fmaf(accH1[j], al_prev[j], __uint_as_float(v1[j]));
        accD4[j] = fmaf(accD4[j], al_prev[j], __uint_as_float(v4[j]));
      }
    };
    auto write_partial = [&](int u) {
      float* rec = sc.part + (size_t)(u + blockIdx.x) * g.rec_stride;
      if (t == 0) {
#pragma unroll
        for (int j = 0; j < GQ; ++j) { rec[j] = m_run[j]; rec[GQ + j] = l_run[j]; }
      }
#pragma unroll
      for (int j = 0; j < GQ; ++j) {
        rec[2 * GQ + j * kHid + t] = accH0[j];
        rec[2 * GQ + j * kHid + 128 + t] = accH1[j];
        rec[2 * GQ + GQ * kHid + j * kDh + t] = accD[j] + accD4[j];
        m_run[j] = -INFINITY; l_run[j] = 0.f; accD[j] = 0.f; accD4[j] = 0.f; accH0[j] = 0.f;
        accH1[j] = 0.f;
      }
    };
    Walk wk;
    init_walk(wk, x0, x1);
    for (int ci = 0; ci < NCH; ++ci) {
      wk.advance_to(ci);
      const int u = wk.u;
      if (u != cur_u) {
        if (cur_u >= 0) {
          fold(ci - 1);                    // the previous unit's last chunk
          if (live) write_partial(cur_u);
        }
        cur_u = u;
      }
      const int st = ci % STAGES, sb = ci & 1, pb = ci & 1;
      live = __all_sync(0xffffffffu, live && mbar_wait(&bar.r_full[st], (ci / STAGES) & 1, abort_flag, err, ERR_TIMEOUT, wlim) &&
                                         mbar_wait(&bar.s_full[sb], (ci >> 1) & 1, abort_flag, err, ERR_TIMEOUT, wlim));
      uint32_t sv[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) sv[j] = 0u;
      if (live) {
        tc_fence_after();
        tmem_ld16(tmem + lane_off + Lay::T_S + sb * 16, sv);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
      }
      const bool valid = t < C;
      float p[GQ], al[GQ];
#pragma unroll
      for (int j = 0; j < GQ; ++j) {
        const float s = valid ? __uint_as_float(sv[j]) : -INFINITY;
        const float mx = warp_max(s);
        if (lane == 0) misc->red_max[w][j] = mx;
        p[j] = s;
      }
      named_bar_sync(1, 128);
#pragma unroll
      for (int j = 0; j < GQ; ++j) {
        const float mc = fmaxf(fmaxf(misc->red_max[0][j], misc->red_max[1][j]),
                               fmaxf(misc->red_max[2][j], misc->red_max[3][j]));
        const float mn = fmaxf(m_run[j], mc);
        al[j] = exp2f(m_run[j] - mn);
        p[j] = exp2f(p[j] - mn);
        m_run[j] = mn;
      }
      // the P and P_res buffers pb were last read by the MMAs of chunk ci-2, whose D3 / D4
      // this group has already folded (so they are complete)
      const int r0 = misc->stage_rec[st][0], r1 = misc->stage_rec[st][1];
      const int nrec = r1 - r0;
      unsigned char* pt = pbase + pb * Lay::P_BUF;
      unsigned char* pr = prbase + pb * Lay::PR_BUF;
      if (valid && live) {
        const int idx = misc->stage_idx[st][t];
#pragma unroll
        for (int j = 0; j < GQ; ++j) {
          *reinterpret_cast<__half*>(pt + kmajor_off(j, t, Lay::P_SBO)) = __float2half_rn(p[j]);
          // P_res: row j, column i = probability of head j at the chunk's i-th flagged token
          if (idx >= 0) st_op16<I8>(pr + kmajor_off(j, idx, Lay::PR_SBO), p[j]);
        }
      }
      if (live && t < kResCap && t >= nrec) {   // columns past the chunk's records
#pragma unroll
        for (int j = 0; j < GQ; ++j)
          st_op16<I8>(pr + kmajor_off(j, t, Lay::PR_SBO), 0.f);
      }
#pragma unroll
      for (int j = 0; j < GQ; ++j) {
        const float s = warp_sum(p[j]);
        if (lane == 0) misc->red_sum[w][j] = s;
      }
      fence_proxy_async_smem();
      named_bar_sync(1, 128);
      if (t == 0 && live) mbar_arrive(&bar.p_ready[pb]);
#pragma unroll
      for (int j = 0; j < GQ; ++j) {
        l_run[j] = l_run[j] * al[j] + misc->red_sum[0][j] + misc->red_sum[1][j] +
                   misc->red_sum[2][j] + misc->red_sum[3][j];
        accD[j] *= al[j];
      }
      // records beyond the first kResCap (rare): CUDA cores, with the rows straight from
      // global memory and the probabilities from the fp16 P tile
      if (live && nrec > kResCap) {
        const uint16_t* rg = reinterpret_cast<const uint16_t*>(cb.res_val);
        const int8_t* rg8 = reinterpret_cast<const int8_t*>(cb.res_val);
        for (int i = kResCap; i < nrec; ++i) {
          const int pos = cb.res_pos[r0 + i];
          if (pos >= C) continue;
          const float dv = I8 ? (float)rg8[(size_t)(r0 + i) * kDh + t] * __half2float(cb.res_scale[r0 + i])
                              : __uint_as_float(((uint32_t)rg[(size_t)(r0 + i) * kDh + t]) << 16);
#pragma unroll
          for (int j = 0; j < GQ; ++j)
            accD[j] = fmaf(__half2float(*reinterpret_cast<const __half*>(pt + kmajor_off(j, pos, Lay::P_SBO))), dv,
                           accD[j]);
        }
      }
      // fold the previous chunk's D3 / D4 when it belongs to this unit (its MMAs ran
      // meanwhile); it is relative to the max after chunk ci-1, so the running sums are
      // rescaled by that chunk's factor first
      if (ci >= 1 && !wk.first_of_unit()) fold(ci - 1);
#pragma unroll
      for (int j = 0; j < GQ; ++j) al_prev[j] = al[j];
    }
    if (NCH > 0) {
      fold(NCH - 1);
      if (live && !*abort_flag && cur_u >= 0) write_partial(cur_u);
    }
  }

  // ------------------------------------------------------------------ teardown
  __syncwarp();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Lay::TMEM_COLS);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

// 2-D bf16 tensor map over a row-major [rows][inner] array, boxes of 64 x box_rows elements
// delivered in the 128-byte swizzle layout.
bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint32_t box_rows) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int R, int C, int GQ, bool I8, bool TW, bool CT>
cudaError_t launch_tc_t(const Geom& g, const CacheBuffers& cb, const Scratch& sc, const void* w1f,
                        cudaStream_t s) {
  using Lay = TcLayout<R, C, I8>;
  const int NG = g.L / g.G;
  const uint64_t rows = (uint64_t)g.B * NG * g.Hkv * g.nLs * C;
  CUtensorMap tmW, tmA, tmQ, tmRes;
  // W1'/2 of every (layer, KV head): [L][Hkv][256][R] 16-bit, boxes of 64 x 128 rows
  if (!make_map(&tmW, w1f, R, (uint64_t)g.L * g.Hkv * kHid, 128)) return cudaErrorInvalidValue;
  if (!make_map(&tmQ, sc.qt_tc, R, (uint64_t)g.U * 16, 16)) return cudaErrorInvalidValue;
  if (I8) {   // int8 rows arrive by plain bulk copies; the tile maps are not used
    tmA = tmQ;
    tmRes = tmQ;
  } else {
    if (!make_map(&tmA, cb.coeff, R, rows, C)) return cudaErrorInvalidValue;
    // the cache keeps kResPad zero rows after its residual rows, so every box is in bounds
    if (!make_map(&tmRes, cb.res_val, kDh, (uint64_t)cb.n_records + kResPad, kResCap))
      return cudaErrorInvalidValue;
  }
  auto k = attend_tc_kernel<R, C, GQ, I8, TW, CT>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::SMEM);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(g.P);
  lc.blockDim = dim3(kThreadsTC);
  lc.dynamicSmemBytes = Lay::SMEM;
  lc.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  // the explicit tile list is read before the set-up: that launch waits for the list's kernel
  lc.attrs = at;
  lc.numAttrs = CT ? 0 : 1;
  return cudaLaunchKernelEx(&lc, k, g, cb, sc, tmW, tmA, tmQ, tmRes);
}

template <int R, int C, int GQ, bool I8>
cudaError_t launch_tc(const Geom& g, const CacheBuffers& cb, const Scratch& sc, const void* w1f,
                      cudaStream_t s) {
  if (sc.tile_total) return launch_tc_t<R, C, GQ, I8, false, true>(g, cb, sc, w1f, s);
  if (g.wait_cycles < kDefaultWaitCycles) return launch_tc_t<R, C, GQ, I8, true, false>(g, cb, sc, w1f, s);
  return launch_tc_t<R, C, GQ, I8, false, false>(g, cb, sc, w1f, s);
}

}  // namespace

// The cache object pads its residual array by kResPad zero rows; callers that pass their
// own arrays (the allocation-free entry point) use the CUDA-core kernels.  The int8 store is
// taken for 128-token chunks.
bool attend_tc_supported(const Geom& g, int dtype, int store) {
  if (dtype != LOWRAM_BF16) return false;
  if (store != LOWRAM_STORE_NATIVE && !(store == LOWRAM_STORE_INT8 && g.C == 128)) return false;
  if (g.d != kDh || g.h != kHid || !(g.g == 4 || g.g == 8)) return false;
  if (!(g.r == 64 || g.r == 128) || !(g.C == 64 || g.C == 128)) return false;
  const uint64_t rows = (uint64_t)g.B * (g.L / g.G) * g.Hkv * g.nLs * g.C;
  if (rows >= (1ull << 31) || (uint64_t)g.U * 16 >= (1ull << 31)) return false;
  return encode_fn() != nullptr;
}

cudaError_t launch_attend_tc(const Geom& g, const CacheBuffers& cb, const Scratch& sc, int store,
                             const void* w1f_tc, int n_sm, cudaStream_t s) {
  (void)n_sm;
  if (cb.n_records + kResPad >= (1ll << 31)) return cudaErrorNotSupported;
  if (store == LOWRAM_STORE_INT8) {
#define LOWRAM_TC_CASE8(RR, GG) \
    if (g.r == RR && g.C == 128 && g.g == GG) return launch_tc<RR, 128, GG, true>(g, cb, sc, w1f_tc, s);
    LOWRAM_TC_CASE8(128, 4)
    LOWRAM_TC_CASE8(64, 4)
    LOWRAM_TC_CASE8(128, 8)
    LOWRAM_TC_CASE8(64, 8)
#undef LOWRAM_TC_CASE8
    return cudaErrorNotSupported;
  }
  if (store != LOWRAM_STORE_NATIVE) return cudaErrorNotSupported;
#define LOWRAM_TC_CASE(RR, CC, GG) \
  if (g.r == RR && g.C == CC && g.g == GG) return launch_tc<RR, CC, GG, false>(g, cb, sc, w1f_tc, s);
  LOWRAM_TC_CASE(128, 128, 4)
  LOWRAM_TC_CASE(128, 64, 4)
  LOWRAM_TC_CASE(64, 128, 4)
  LOWRAM_TC_CASE(64, 64, 4)
  LOWRAM_TC_CASE(128, 128, 8)
  LOWRAM_TC_CASE(128, 64, 8)
  LOWRAM_TC_CASE(64, 128, 8)
  LOWRAM_TC_CASE(64, 64, 8)
#undef LOWRAM_TC_CASE
  return cudaErrorNotSupported;
}

}  // namespace lowram
