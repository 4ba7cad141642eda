// C ABI of the LowRAM decode library: cache object, argument checks, launches.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "lowram_internal.cuh"
#include "upkeep.cuh"
#include "reuse.cuh"

using namespace lowram;

struct lowram_cache {
  lowram_config cfg;
  int nC, nL, NG, g, device, n_sm;
  int nLs, nCs;                // per-unit capacity (strides) in live slots / chunk ids
  bool canonical;              // records laid out unit by unit in unit order, with slack
  bool last_repack_in_place;
  void* up_mem;                // re-pack scratch (encoder inputs, outputs and workspace), kept
  size_t up_bytes;
  bool up_w2h_ready;           // the re-pack scratch's encoder workspace holds W2 in fp16
  // lowram_decode_attn_host replays its decode (on the staging buffers) from a CUDA graph
  // captured at its first call for a layer range; a re-pack or destroy drops it
  cudaStream_t cap_stream;
  cudaGraphExec_t host_exec;
  int hg_layer0, hg_n, hg_sel;
  bool hg_off;                 // capture failed once: eager calls from then on
  size_t s_dt;                 // bytes of one dt element
  void* owned[48];             // every device allocation the cache owns
  int n_owned;
  CacheBuffers cb;
  float* w1f_t;                // [L][Hkv][r][h] fp32 fold for the CUDA-core path
  void* w1f_tc;                // [L][Hkv][h][r] 16-bit fold / 2 for the tensor-core path
  Scratch sc;
  size_t part_floats;          // capacity of sc.part
  void* q_stage;               // host entry point staging
  void* out_stage;
  int32_t* sel_stage;
  cudaEvent_t ev[4];
  bool ev_on;
  int last_launches, last_path;
  long long wait_limit;        // main-loop wait limit of the tensor-core kernel (test hook)
  // context-sharded decode: tile list of phase 2, and the layer range phase 1 prepared
  int32_t *t_unit, *t_slot, *t_ptr, *t_total, *t_cnt;
  int shard_l0, shard_n;
  uint64_t generation;         // advanced by every re-pack (a reuse store is tied to one)
};

// A store of rebuilt chunk values tied to one cache (reuse.cu has the kernels).
struct lowram_reuse {
  lowram_cache* cache;
  uint64_t generation;
  ReuseDev d;
  void* mem[12];
  int n_mem;
};

namespace {

thread_local std::string g_last_error;

lowram_status cuda_fail(cudaError_t e, const char* where) {
  g_last_error = std::string(where) + ": " + cudaGetErrorString(e);
  return LOWRAM_ECUDA;
}

lowram_status inval(const char* why) {
  g_last_error = why;
  return LOWRAM_EINVAL;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

lowram_status check_config(const lowram_config* c) {
  if (!c) return inval("config is NULL");
  if (c->batch < 1 || c->n_layers < 1 || c->group < 1 || c->n_kv_heads < 1 || c->n_q_heads < 1 ||
      c->head_dim < 1 || c->rank < 1 || c->mlp_hidden < 1 || c->n_ctx < 1 || c->chunk < 1 ||
      c->top_k < 1 || c->tail_cap < 0 || c->n_live < 1)
    return inval("config sizes must be positive");
  if (c->n_layers % c->group) return inval("n_layers must be a multiple of group");
  if (c->n_q_heads % c->n_kv_heads) return inval("n_q_heads must be a multiple of n_kv_heads");
  if (c->n_ctx % c->chunk) return inval("n_ctx must be a multiple of chunk");
  const int nC = c->n_ctx / c->chunk;
  if (c->n_live > nC) return inval("n_live exceeds the number of chunks");
  if (c->top_k > c->n_live) return inval("top_k exceeds the live chunks");
  if (c->rank > c->group * c->head_dim) return inval("rank exceeds group * head_dim");
  if (c->chunk > 32767) return inval("chunk exceeds 32767");
  if (c->n_q_heads / c->n_kv_heads > kMaxG) return inval("more than 16 query heads per KV head");
  if (c->head_dim > kMaxD || c->rank > kMaxR || c->mlp_hidden > kMaxH)
    return inval("head_dim/rank/mlp_hidden above the supported maximum (256/512/1024)");
  if (nC > kMaxChunks) return inval("more than 8192 chunks");
  // the kernels index coefficient rows with 32-bit integers
  if ((uint64_t)c->batch * (uint64_t)(c->n_layers / c->group) * (uint64_t)c->n_kv_heads * (uint64_t)c->n_live *
          (uint64_t)c->chunk >= (1ull << 31))
    return inval("coefficient rows batch * (n_layers / group) * n_kv_heads * n_live * chunk must stay below 2^31");
  if (c->tail_cap > kMaxTail) return inval("tail_cap exceeds 4096");
  if (c->dtype != LOWRAM_F32 && c->dtype != LOWRAM_BF16) return inval("unknown dtype");
  if (c->store != LOWRAM_STORE_NATIVE && c->store != LOWRAM_STORE_INT8) return inval("unknown store");
  if (c->store == LOWRAM_STORE_INT8 && c->dtype != LOWRAM_BF16) return inval("int8 store needs BF16");
  return LOWRAM_OK;
}

void fill_bytes(const lowram_config* c, int64_t n_records, bool has_slot, lowram_bytes* b) {
  const uint64_t B = c->batch, L = c->n_layers, G = c->group, H = c->n_kv_heads;
  const uint64_t d = c->head_dim, r = c->rank, h = c->mlp_hidden, N = c->n_ctx, C = c->chunk;
  const uint64_t T = c->tail_cap, nC = N / C, nL = c->n_live, NG = L / G;
  const uint64_t s = c->dtype == LOWRAM_F32 ? 4 : 2;
  const bool i8 = c->store == LOWRAM_STORE_INT8;
  const uint64_t sa = i8 ? 1 : s;
  const uint64_t R = (uint64_t)n_records;
  b->coeff = B * NG * H * nL * C * (r * sa + (i8 ? 2 : 0));
  b->basis = L * H * r * d * s;
  b->predictor = 2 * L * H * h * d * s;
  b->summary = B * NG * H * nL * r * s;
  b->residual = R * (d * sa + 2 + (i8 ? 2 : 0)) + B * L * H * (nL + 1) * 4;
  b->index = has_slot ? B * NG * H * nC * 2 : 0;
  const uint64_t st = i8 ? 2 : s;
  b->tail = 2 * B * L * H * T * d * st + 4 * B;
  b->total = b->coeff + b->basis + b->predictor + b->summary + b->residual + b->index + b->tail;
  b->dense_equiv = lowram_dense_kv_bytes(c->n_layers, c->n_kv_heads, c->head_dim, c->n_ctx,
                                         (int32_t)s, c->batch) +
                   2 * B * L * H * T * d * s;
}

Geom make_geom(const lowram_cache* c, int layer0, int n_layers, bool tc) {
  Geom g;
  const lowram_config& f = c->cfg;
  g.B = f.batch; g.L = f.n_layers; g.G = f.group; g.Hkv = f.n_kv_heads; g.Hq = f.n_q_heads;
  g.g = f.n_q_heads / f.n_kv_heads; g.d = f.head_dim; g.r = f.rank; g.h = f.mlp_hidden;
  g.N = f.n_ctx; g.C = f.chunk; g.nC = c->nC; g.nL = c->nL; g.k = f.top_k; g.T = f.tail_cap;
  g.nLs = c->nLs; g.nCs = c->nCs;
  g.layer0 = layer0; g.n_layers = n_layers;
  g.U = n_layers * g.Hkv * g.B;
  const long long total = (long long)g.U * g.k;
  const long long pmax = tc ? c->n_sm : 4LL * c->n_sm;
  g.P = (int)(total < pmax ? total : pmax);
  g.rec_stride = (2 * g.g + g.g * g.h + g.g * g.d + 3) & ~3;
  g.tail_stride = (2 * g.g + g.g * g.d + 3) & ~3;
  g.max_rec = max_records_per_unit(total, g.P, g.k);
  g.qk_scale_log2 = 1.4426950408889634f / sqrtf((float)g.d);
  g.wait_cycles = c->wait_limit;
  return g;
}

// Test hook (lowram_debug_fail_alloc): allocations still to succeed before one fails, or -1.
std::atomic<int> g_fail_after{-1};

// Every device allocation of the library goes through here.
cudaError_t device_malloc(void** p, size_t bytes) {
  int n = g_fail_after.load();
  while (n >= 0) {
    if (g_fail_after.compare_exchange_weak(n, n - 1)) {
      if (n == 0) {   // the injected failure (the hook is now off again: the counter is -1)
        *p = nullptr;
        return cudaErrorMemoryAllocation;
      }
      break;
    }
  }
  return cudaMalloc(p, bytes);
}

template <typename P>
lowram_status alloc(lowram_cache* c, P** out, size_t bytes) {
  void* p = nullptr;
  if (bytes == 0) bytes = 16;
  if (c->n_owned >= (int)(sizeof(c->owned) / sizeof(c->owned[0]))) {
    g_last_error = "internal: too many owned allocations";
    return LOWRAM_ENOMEM;
  }
  cudaError_t e = device_malloc(&p, bytes);
  if (e != cudaSuccess) {
    g_last_error = std::string("cudaMalloc: ") + cudaGetErrorString(e);
    return LOWRAM_ENOMEM;
  }
  c->owned[c->n_owned++] = p;
  *out = static_cast<P*>(p);
  return LOWRAM_OK;
}

}  // namespace

namespace lowram {
// Sets the calling thread's text returned by lowram_last_error_string (for other files).
void set_last_error(const char* msg) { g_last_error = msg; }
}  // namespace lowram

extern "C" {

uint64_t lowram_dense_kv_bytes(int32_t n_layers, int32_t n_kv_heads, int32_t head_dim,
                               int64_t n_ctx, int32_t bytes_per_scalar, int32_t batch) {
  if (n_layers < 0 || n_kv_heads < 0 || head_dim < 0 || n_ctx < 0 || bytes_per_scalar < 0 ||
      batch < 0)
    return 0;
  return 2ull * (uint64_t)n_layers * (uint64_t)n_kv_heads * (uint64_t)head_dim *
         (uint64_t)n_ctx * (uint64_t)bytes_per_scalar * (uint64_t)batch;
}

lowram_status lowram_config_bytes(const lowram_config* cfg, int64_t n_records, int32_t has_slot,
                                  lowram_bytes* out) {
  lowram_status st = check_config(cfg);
  if (st != LOWRAM_OK) return st;
  if (!out || n_records < 0) return inval("bad n_records or NULL output");
  fill_bytes(cfg, n_records, has_slot != 0 && cfg->n_live < cfg->n_ctx / cfg->chunk, out);
  return LOWRAM_OK;
}

const char* lowram_status_string(lowram_status s) {
  switch (s) {
    case LOWRAM_OK: return "ok";
    case LOWRAM_EINVAL: return "invalid argument";
    case LOWRAM_ENOMEM: return "out of device memory";
    case LOWRAM_ECUDA: return "CUDA error";
    case LOWRAM_EUNSUPPORTED: return "unsupported shapes for the requested path";
    case LOWRAM_ECORRUPT: return "inconsistent cache tables";
    case LOWRAM_ETIMEOUT: return "a kernel gave up a bounded wait";
  }
  return "unknown status";
}

const char* lowram_last_error_string(void) { return g_last_error.c_str(); }

// ------------------------------------------------------------------------------ encoder

namespace {

lowram_status encode_geom(const lowram_config* cfg, Geom* g) {
  if (!cfg) return inval("config is NULL");
  // top_k, n_q_heads and tail_cap play no part in encoding: check the rest
  lowram_config cc = *cfg;
  cc.top_k = 1;
  cc.n_q_heads = cc.n_kv_heads;
  cc.tail_cap = 0;
  const lowram_config* c = &cc;
  lowram_status st = check_config(c);
  if (st != LOWRAM_OK) return st;
  const int nC = c->n_ctx / c->chunk;
  if (c->n_live != nC) return inval("the encoder evicts nothing: n_live must equal n_ctx / chunk");
  if (c->dtype != LOWRAM_BF16 || c->head_dim != 128 || c->mlp_hidden != 256 || !(c->rank == 64 || c->rank == 128) ||
      !(c->chunk == 64 || c->chunk == 128)) {
    g_last_error = "the encoder takes bf16, head_dim 128, mlp_hidden 256, rank 64 or 128, chunk 64 or 128";
    return LOWRAM_EUNSUPPORTED;
  }
  *g = Geom{};
  g->B = c->batch; g->L = c->n_layers; g->G = c->group; g->Hkv = c->n_kv_heads; g->Hq = c->n_q_heads;
  g->g = c->n_q_heads / c->n_kv_heads; g->d = c->head_dim; g->r = c->rank; g->h = c->mlp_hidden;
  g->N = c->n_ctx; g->C = c->chunk; g->nC = nC; g->nL = nC; g->k = c->top_k; g->T = c->tail_cap;
  g->nLs = nC; g->nCs = nC;
  g->layer0 = 0; g->n_layers = c->n_layers;
  g->wait_cycles = kDefaultWaitCycles;
  return LOWRAM_OK;
}

}  // namespace

uint64_t lowram_encode_workspace_bytes(const lowram_config* cfg) {
  Geom g;
  if (encode_geom(cfg, &g) != LOWRAM_OK) return 0;
  return encode_workspace_bytes(g);
}

lowram_status lowram_encode(const lowram_config* cfg, int32_t n_resid, const void* keys, const void* values,
                            const void* basis, const void* w1, const void* w2, const lowram_encode_dst* dst,
                            void* workspace, uint64_t workspace_bytes, lowram_stream stream) {
  Geom g;
  lowram_status st = encode_geom(cfg, &g);
  if (st != LOWRAM_OK) return st;
  if (n_resid < 0 || n_resid > g.N) return inval("n_resid must lie in [0, n_ctx]");
  const long long units = (long long)g.B * g.L * g.Hkv;
  if (units * n_resid >= (1LL << 31)) return inval("B * L * Hkv * n_resid must be below 2^31");
  if (!dst) return inval("NULL destination");
  const void* req[] = {keys, values, basis, w1, w2, dst->coeff, dst->summary, dst->res_ptr, workspace};
  for (const void* p : req)
    if (!p || !aligned16(p)) return inval("a required pointer is NULL or not 16-byte aligned");
  const bool i8 = cfg->store == LOWRAM_STORE_INT8;
  if (i8 && (!dst->coeff_scale || !aligned16(dst->coeff_scale)))
    return inval("int8 store needs a 16-byte aligned coeff_scale");
  if (n_resid > 0) {
    if (!dst->res_pos || !aligned16(dst->res_pos) || !dst->res_val || !aligned16(dst->res_val))
      return inval("residual arrays missing or misaligned");
    if (i8 && (!dst->res_scale || !aligned16(dst->res_scale))) return inval("int8 store needs res_scale");
  }
  if (workspace_bytes < encode_workspace_bytes(g)) return inval("workspace smaller than lowram_encode_workspace_bytes");
  cudaError_t e = launch_encode(g, cfg->store, n_resid, keys, values, basis, w1, w2, *dst, workspace,
                                reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "encode");
  return LOWRAM_OK;
}

lowram_status lowram_cache_create(const lowram_config* cfg, const lowram_cache_src* src,
                                  lowram_cache** out, lowram_stream stream) {
  lowram_status st = check_config(cfg);
  if (st != LOWRAM_OK) return st;
  if (!src || !out) return inval("NULL src or out");
  *out = nullptr;
  const bool i8 = cfg->store == LOWRAM_STORE_INT8;
  const int nC = cfg->n_ctx / cfg->chunk;
  const bool evict = cfg->n_live < nC;
  const void* need[] = {src->coeff, src->basis, src->w1, src->w2, src->summary, src->res_ptr,
                        src->tail_k, src->tail_v, src->tail_len};
  for (const void* p : need)
    if (!p || !aligned16(p)) return inval("a required source pointer is NULL or not 16-byte aligned");
  if (src->n_records < 0 || src->n_records >= (1LL << 31)) return inval("n_records out of range");
  if (src->n_records > 0 && (!src->res_pos || !src->res_val || !aligned16(src->res_val) ||
                             !aligned16(src->res_pos)))
    return inval("residual arrays missing or misaligned");
  if (i8 && (!src->coeff_scale || !aligned16(src->coeff_scale) ||
             (src->n_records > 0 && (!src->res_scale || !aligned16(src->res_scale)))))
    return inval("int8 store needs coeff_scale and res_scale");
  if (evict && (!src->slot || !aligned16(src->slot))) return inval("eviction needs a slot map");

  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  int n_sm = 0;
  e = cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");

  lowram_cache* c = new lowram_cache();
  std::memset(c, 0, sizeof(*c));
  c->cfg = *cfg;
  c->nC = nC; c->nL = cfg->n_live; c->NG = cfg->n_layers / cfg->group;
  c->nLs = c->nL; c->nCs = nC; c->canonical = false; c->last_repack_in_place = false;
  c->up_mem = nullptr; c->up_bytes = 0; c->up_w2h_ready = false;
  c->cap_stream = nullptr; c->host_exec = nullptr; c->hg_off = false;
  c->g = cfg->n_q_heads / cfg->n_kv_heads;
  c->device = dev; c->n_sm = n_sm;
  c->s_dt = cfg->dtype == LOWRAM_F32 ? 4 : 2;
  c->wait_limit = kDefaultWaitCycles;

  const size_t B = cfg->batch, L = cfg->n_layers, H = cfg->n_kv_heads, d = cfg->head_dim;
  const size_t r = cfg->rank, h = cfg->mlp_hidden, C = cfg->chunk, T = cfg->tail_cap;
  const size_t nL = cfg->n_live, NG = c->NG, R = (size_t)src->n_records, s = c->s_dt;
  const size_t sa = i8 ? 1 : s, st16 = i8 ? 2 : s;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);

  struct Item { const void* from; void** to; size_t bytes; };
  void* p_coeff = nullptr; void* p_cscale = nullptr; void* p_basis = nullptr; void* p_w1 = nullptr;
  void* p_w2 = nullptr; void* p_summ = nullptr; void* p_slot = nullptr; void* p_rptr = nullptr;
  void* p_rpos = nullptr; void* p_rval = nullptr; void* p_rscale = nullptr; void* p_tk = nullptr;
  void* p_tv = nullptr; void* p_tl = nullptr;
  Item items[] = {
      {src->coeff, &p_coeff, B * NG * H * nL * C * r * sa},
      {i8 ? src->coeff_scale : nullptr, &p_cscale, i8 ? B * NG * H * nL * C * 2 : 0},
      {src->basis, &p_basis, L * H * r * d * s},
      {src->w1, &p_w1, L * H * h * d * s},
      {src->w2, &p_w2, L * H * d * h * s},
      {src->summary, &p_summ, B * NG * H * nL * r * s},
      {evict ? src->slot : nullptr, &p_slot, evict ? B * NG * H * nC * 2 : 0},
      {src->res_ptr, &p_rptr, B * L * H * (nL + 1) * 4},
      {R ? src->res_pos : nullptr, &p_rpos, R * 2},
      {(i8 && R) ? src->res_scale : nullptr, &p_rscale, (i8 && R) ? R * 2 : 0},
      {src->tail_k, &p_tk, B * L * H * T * d * st16},
      {src->tail_v, &p_tv, B * L * H * T * d * st16},
      {src->tail_len, &p_tl, B * 4},
  };
  for (Item& it : items) {
    if (!it.from) continue;
    st = alloc(c, it.to, it.bytes);
    if (st != LOWRAM_OK) { lowram_cache_destroy(c); return st; }
    if (it.bytes) {
      e = cudaMemcpyAsync(*it.to, it.from, it.bytes, cudaMemcpyDeviceToDevice, cs);
      if (e != cudaSuccess) { lowram_cache_destroy(c); return cuda_fail(e, "cudaMemcpyAsync"); }
    }
  }
  // residual rows, followed by kResPad zero rows: the tensor-core kernel loads a fixed box
  // of kResPad rows from each chunk's first record, so the box never leaves the array
  if ((st = alloc(c, &p_rval, (R + kResPad) * d * sa)) != LOWRAM_OK) { lowram_cache_destroy(c); return st; }
  if (R) {
    e = cudaMemcpyAsync(p_rval, src->res_val, R * d * sa, cudaMemcpyDeviceToDevice, cs);
    if (e != cudaSuccess) { lowram_cache_destroy(c); return cuda_fail(e, "cudaMemcpyAsync"); }
  }
  e = cudaMemsetAsync(static_cast<unsigned char*>(p_rval) + R * d * sa, 0, kResPad * d * sa, cs);
  if (e != cudaSuccess) { lowram_cache_destroy(c); return cuda_fail(e, "cudaMemsetAsync"); }
  c->cb.coeff = p_coeff; c->cb.coeff_scale = static_cast<const __half*>(p_cscale);
  c->cb.basis = p_basis; c->cb.w1 = p_w1; c->cb.w2 = p_w2; c->cb.summary = p_summ;
  c->cb.slot = static_cast<const int16_t*>(p_slot);
  c->cb.res_ptr = static_cast<const int32_t*>(p_rptr);
  c->cb.res_pos = static_cast<const uint16_t*>(p_rpos);
  c->cb.res_val = p_rval; c->cb.res_scale = static_cast<const __half*>(p_rscale);
  c->cb.tail_k = p_tk; c->cb.tail_v = p_tv; c->cb.tail_len = static_cast<const int32_t*>(p_tl);
  c->cb.n_records = src->n_records;

  // folded predictor weights
  Geom gall = make_geom(c, 0, cfg->n_layers, false);
  if ((st = alloc(c, &c->w1f_t, L * H * r * h * 4)) != LOWRAM_OK) { lowram_cache_destroy(c); return st; }
  if (cfg->dtype == LOWRAM_BF16) {
    if ((st = alloc(c, &c->w1f_tc, L * H * h * r * 2)) != LOWRAM_OK) { lowram_cache_destroy(c); return st; }
  }
  e = launch_fold(gall, c->cb, cfg->dtype, cfg->store, c->w1f_t, c->w1f_tc, cs);
  if (e != cudaSuccess) { lowram_cache_destroy(c); return cuda_fail(e, "fold"); }

  // scratch for an all-layer call
  const size_t Umax = L * H * B;
  const size_t g = c->g, k = cfg->top_k;
  const size_t rec_stride = (2 * g + g * h + g * d + 3) & ~size_t(3);
  const size_t tail_stride = (2 * g + g * d + 3) & ~size_t(3);
  c->part_floats = (Umax + 4 * (size_t)n_sm + 1) * rec_stride;
  if ((st = alloc(c, &c->sc.qt, Umax * g * r * 4)) != LOWRAM_OK ||
      (st = alloc(c, &c->sc.qt_tc, Umax * 16 * r * 2)) != LOWRAM_OK ||
      (st = alloc(c, &c->sc.sel_slot, Umax * k * 4)) != LOWRAM_OK ||
      (st = alloc(c, &c->sc.sel_id, Umax * k * 4)) != LOWRAM_OK ||
      (st = alloc(c, &c->sc.part, c->part_floats * 4)) != LOWRAM_OK ||
      (st = alloc(c, &c->sc.tail_part, Umax * tail_stride * 4)) != LOWRAM_OK ||
      (st = alloc(c, &c->sc.err, 16)) != LOWRAM_OK ||
      (st = alloc(c, &c->q_stage, L * B * cfg->n_q_heads * d * s)) != LOWRAM_OK ||
      (st = alloc(c, &c->out_stage, L * B * cfg->n_q_heads * d * s)) != LOWRAM_OK ||
      (st = alloc(c, &c->sel_stage, Umax * k * 4)) != LOWRAM_OK ||
      (st = alloc(c, &c->t_unit, Umax * k * 4)) != LOWRAM_OK ||
      (st = alloc(c, &c->t_slot, Umax * k * 4)) != LOWRAM_OK ||
      (st = alloc(c, &c->t_ptr, (Umax + 1) * 4)) != LOWRAM_OK ||
      (st = alloc(c, &c->t_total, 16)) != LOWRAM_OK ||
      (st = alloc(c, &c->t_cnt, Umax * 4)) != LOWRAM_OK) {
    lowram_cache_destroy(c);
    return st;
  }
  e = cudaMemsetAsync(c->sc.err, 0, 16, cs);
  if (e != cudaSuccess) { lowram_cache_destroy(c); return cuda_fail(e, "cudaMemsetAsync"); }
  e = cudaMemsetAsync(c->sc.qt_tc, 0, Umax * 16 * r * 2, cs);
  if (e != cudaSuccess) { lowram_cache_destroy(c); return cuda_fail(e, "cudaMemsetAsync"); }
  c->last_path = -1;
  c->shard_l0 = -1;
  c->shard_n = 0;
  *out = c;
  return LOWRAM_OK;
}

void lowram_cache_destroy(lowram_cache* c) {
  if (!c) return;
  cudaDeviceSynchronize();
  for (int i = 0; i < c->n_owned; ++i) cudaFree(c->owned[i]);
  if (c->up_mem) cudaFree(c->up_mem);
  if (c->host_exec) cudaGraphExecDestroy(c->host_exec);
  if (c->cap_stream) cudaStreamDestroy(c->cap_stream);
  delete c;
}

lowram_status lowram_cache_bytes(const lowram_cache* c, lowram_bytes* out) {
  if (!c || !out) return inval("NULL cache or output");
  fill_bytes(&c->cfg, c->cb.n_records, c->cb.slot != nullptr, out);
  return LOWRAM_OK;
}

lowram_status lowram_cache_view(const lowram_cache* c, lowram_config* cfg, lowram_cache_src* src,
                                int32_t* spare_chunks) {
  if (!c || !cfg || !src || !spare_chunks) return inval("NULL cache or output");
  *spare_chunks = c->nLs - c->nL;
  *cfg = c->cfg;
  src->coeff = c->cb.coeff; src->coeff_scale = c->cb.coeff_scale; src->basis = c->cb.basis;
  src->w1 = c->cb.w1; src->w2 = c->cb.w2; src->summary = c->cb.summary; src->slot = c->cb.slot;
  src->res_ptr = c->cb.res_ptr; src->res_pos = c->cb.res_pos; src->res_val = c->cb.res_val;
  src->res_scale = c->cb.res_scale; src->tail_k = c->cb.tail_k; src->tail_v = c->cb.tail_v;
  src->tail_len = c->cb.tail_len; src->n_records = c->cb.n_records;
  return LOWRAM_OK;
}

lowram_status lowram_cache_append(lowram_cache* c, const void* k_new, const void* v_new, lowram_stream stream) {
  if (!c) return inval("NULL cache");
  if (!k_new || !v_new || !aligned16(k_new) || !aligned16(v_new))
    return inval("k_new / v_new NULL or not 16-byte aligned");
  if (c->cfg.tail_cap < 1) return inval("the cache has no tail (tail_cap = 0)");
  const size_t eb = c->cfg.store == LOWRAM_STORE_INT8 ? 2 : c->s_dt;
  const size_t row = (size_t)c->cfg.head_dim * eb;
  if (row % 16) {
    g_last_error = "append moves 16-byte pieces: head_dim * element size must be a multiple of 16";
    return LOWRAM_EUNSUPPORTED;
  }
  cudaError_t e = launch_append(c->cfg.batch, c->cfg.n_layers, c->cfg.n_kv_heads, c->cfg.tail_cap, (int)row, k_new,
                                v_new, const_cast<void*>(c->cb.tail_k), const_cast<void*>(c->cb.tail_v),
                                const_cast<int32_t*>(c->cb.tail_len), c->sc.err, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "append");
  return LOWRAM_OK;
}

}  // extern "C"

namespace {

// Device allocations of one re-pack; whatever is not handed to the cache is freed on exit.
struct RepackMem {
  std::vector<void*> ptrs;
  ~RepackMem() {
    for (void* p : ptrs) cudaFree(p);
  }
  template <typename P>
  lowram_status get(P** out, size_t bytes) {
    void* p = nullptr;
    cudaError_t e = device_malloc(&p, bytes ? bytes : 16);
    if (e != cudaSuccess) {
      g_last_error = std::string("cudaMalloc: ") + cudaGetErrorString(e);
      return LOWRAM_ENOMEM;
    }
    ptrs.push_back(p);
    *out = static_cast<P*>(p);
    return LOWRAM_OK;
  }
  void release(const void* p) {   // the cache owns it from now on
    for (auto& q : ptrs)
      if (q == p) q = nullptr;
  }
};

// new_p replaces old_p among the cache's allocations (old_p is freed); an array the cache
// did not hold before (no records at create time) is added.
void swap_owned(lowram_cache* c, const void* old_p, void* new_p) {
  if (old_p)
    for (int i = 0; i < c->n_owned; ++i)
      if (c->owned[i] == old_p) {
        cudaFree(c->owned[i]);
        c->owned[i] = new_p;
        return;
      }
  c->owned[c->n_owned++] = new_p;
}

// The re-pack scratch, carved from one allocation (256-byte aligned pieces): the error
// words, the encoder's workspace, the gathered tail chunk (when T > C) and the encoder's
// outputs.
struct UpScratch {
  uint32_t* err;
  void* kg;
  void* vg;
  lowram_encode_dst dst;
  void* ws;
};

size_t carve_up(void* base, size_t gather, size_t coeff, size_t cscale, size_t summ, size_t rptr, size_t rpos,
                size_t rval, size_t rscale, size_t ws, UpScratch* o) {
  size_t off = 0;
  auto take = [&](size_t n) -> void* {
    void* p = base ? static_cast<unsigned char*>(base) + off : nullptr;
    off += (n + 255) & ~size_t(255);
    return n ? p : nullptr;
  };
  o->err = static_cast<uint32_t*>(take(16));
  o->ws = take(ws);   // at a fixed offset: the fp16 W2 it keeps between re-packs stays put
  o->kg = take(gather);
  o->vg = take(gather);
  o->dst.coeff = take(coeff);
  o->dst.coeff_scale = take(cscale);
  o->dst.summary = take(summ);
  o->dst.res_ptr = static_cast<int32_t*>(take(rptr));
  o->dst.res_pos = static_cast<uint16_t*>(take(rpos));
  o->dst.res_val = take(rval);
  o->dst.res_scale = take(rscale);
  return off;
}

}  // namespace

extern "C" {

lowram_status lowram_cache_repack(lowram_cache* c, int32_t n_resid, lowram_stream stream) {
  if (!c) return inval("NULL cache");
  c->shard_l0 = -1;
  const lowram_config f = c->cfg;
  const int C = f.chunk, T = f.tail_cap;
  if (n_resid < 0 || n_resid > C) return inval("n_resid must lie in [0, chunk]");
  if (T < C) return inval("the tail cannot hold a chunk (tail_cap < chunk)");
  if (c->nC + 1 > kMaxChunks || (long long)f.n_ctx + C >= (1LL << 31)) return inval("the cache is at its chunk limit");
  // the new chunk is encoded by the encoder kernels: their shapes
  lowram_config ec = f;
  ec.n_ctx = C;
  ec.n_live = 1;
  Geom ge;
  lowram_status st = encode_geom(&ec, &ge);
  if (st != LOWRAM_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t B = f.batch, L = f.n_layers, H = f.n_kv_heads, d = f.head_dim, r = f.rank;
  const size_t NG = c->NG, nC = c->nC, nL = c->nL, U = B * L * H;
  const size_t nLs = c->nLs, nCs = c->nCs;
  const bool i8 = f.store == LOWRAM_STORE_INT8;
  const size_t sa = i8 ? 1 : 2, tail_row = d * 2, n_new = U * (size_t)n_resid;

  RepackMem m;
  // scratch kept by the cache between re-packs (grown when this call needs more)
  UpScratch up;
  auto carve = [&](void* base) {
    return carve_up(base, T != C ? U * C * tail_row : 0, B * NG * H * C * r * sa, i8 ? B * NG * H * C * 2 : 0,
                    B * NG * H * r * 2, U * 2 * 4, n_new * 2, n_new * d * sa, i8 ? n_new * 2 : 0,
                    encode_workspace_bytes(ge, true), &up);
  };
  const size_t up_need = carve(nullptr);
  if (up_need > c->up_bytes) {
    if (c->up_mem) cudaFree(c->up_mem);
    c->up_mem = nullptr;
    c->up_bytes = 0;
    c->up_w2h_ready = false;
    cudaError_t ea = device_malloc(&c->up_mem, up_need);
    if (ea != cudaSuccess) {
      c->up_mem = nullptr;
      g_last_error = std::string("cudaMalloc: ") + cudaGetErrorString(ea);
      return LOWRAM_ENOMEM;
    }
    c->up_bytes = up_need;
  }
  carve(c->up_mem);
  uint32_t* err = up.err;
  cudaError_t e = cudaMemsetAsync(err, 0, 16, s);
  // 1. every tail must hold a chunk; room for the chunk in place?
  const bool room_slots = c->canonical && nL + 1 <= nLs && nC + 1 <= nCs;
  if (e == cudaSuccess && room_slots)
    e = launch_repack_room((int)U, (int)nL, (int)nLs, n_resid, c->cb.res_ptr, c->cb.n_records, err + 1, s);
  std::vector<int32_t> tl(B);
  uint32_t no_room = 0;
  if (e == cudaSuccess) e = cudaMemcpyAsync(tl.data(), c->cb.tail_len, B * 4, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(&no_room, err + 1, 4, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "read tail lengths");
  for (size_t b = 0; b < B; ++b)
    if (tl[b] < C || tl[b] > T) return inval("every sequence's tail must hold at least one chunk");
  const bool in_place = room_slots && !no_room;

  // 2. the oldest C tail tokens as dense [B][L][Hkv][C][d] keys and values
  const void* keys = c->cb.tail_k;
  const void* vals = c->cb.tail_v;
  if (T != C) {
    void *kg = up.kg, *vg = up.vg;
    e = cudaMemcpy2DAsync(kg, C * tail_row, c->cb.tail_k, (size_t)T * tail_row, C * tail_row, U, cudaMemcpyDeviceToDevice, s);
    if (e == cudaSuccess)
      e = cudaMemcpy2DAsync(vg, C * tail_row, c->cb.tail_v, (size_t)T * tail_row, C * tail_row, U, cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess) return cuda_fail(e, "gather the tail's oldest chunk");
    keys = kg;
    vals = vg;
  }
  // 3. encode it
  const lowram_encode_dst dst = up.dst;
  void* ws = up.ws;
  // the cache's own folds of W1 (the encoder would compute the same), and W2 in fp16 kept
  // in the scratch from the previous re-pack
  e = launch_encode(ge, f.store, n_resid, keys, vals, c->cb.basis, c->cb.w1, c->cb.w2, dst, ws, s, c->w1f_t,
                    c->w1f_tc, c->up_w2h_ready);
  if (e != cudaSuccess) return cuda_fail(e, "encode the new chunk");
  c->up_w2h_ready = true;

  // 2-D copy of B*NG*H rows: `width` bytes from `from` (pitch spitch) to `to` (pitch dpitch)
  auto rows2d = [&](void* to, size_t dpitch, const void* from, size_t spitch, size_t width) {
    return cudaMemcpy2DAsync(to, dpitch, from, spitch, width, B * NG * H, cudaMemcpyDeviceToDevice, s);
  };
  auto at = [](const void* p, size_t off) { return static_cast<unsigned char*>(const_cast<void*>(p)) + off; };
  long long total = c->cb.n_records;
  void *coeff = nullptr, *cscale = nullptr, *summ = nullptr, *rval = nullptr;
  int16_t* slot = nullptr;
  int32_t* rptr = nullptr;
  uint16_t* rpos = nullptr;
  __half* rscale = nullptr;
  size_t nLs2 = nLs, nCs2 = nCs;
  if (in_place) {
    // 4a. the new chunk into slot nL of every unit; records after each unit's last ones
    e = rows2d(at(c->cb.coeff, nL * C * r * sa), nLs * C * r * sa, dst.coeff, C * r * sa, C * r * sa);
    if (e == cudaSuccess && i8)
      e = rows2d(at(c->cb.coeff_scale, nL * C * 2), nLs * C * 2, dst.coeff_scale, C * 2, C * 2);
    if (e == cudaSuccess) e = rows2d(at(c->cb.summary, nL * r * 2), nLs * r * 2, dst.summary, r * 2, r * 2);
    if (e == cudaSuccess && c->cb.slot)
      e = launch_repack_slot((long long)(B * NG * H), (int)nCs, (int)nC, (int)nL, const_cast<int16_t*>(c->cb.slot), s);
    if (e == cudaSuccess)
      e = launch_repack_append_records((int)U, (int)nL, (int)nLs, (int)(d * sa), c->cb.n_records, (long long)n_new,
                                       dst.res_ptr, dst.res_pos, dst.res_val, static_cast<const __half*>(dst.res_scale),
                                       const_cast<int32_t*>(c->cb.res_ptr), const_cast<uint16_t*>(c->cb.res_pos),
                                       const_cast<void*>(c->cb.res_val), const_cast<__half*>(c->cb.res_scale), err, s);
    if (e != cudaSuccess) return cuda_fail(e, "write the new chunk in place");
  } else {
    // 4b. arrays of the longer cache with spare capacity: old rows, then the new chunk's,
    // per (b, group, KV head); spare chunks and spare records per unit for later re-packs
    const size_t spare = std::max<size_t>(kSpareChunksMin, (nL + 1) / kSpareChunksDiv);
    nLs2 = nL + 1 + spare;
    nCs2 = nC + 1 + spare;
    if (nCs2 > (size_t)kMaxChunks) nCs2 = nC + 1, nLs2 = nL + 1;   // no room to spare
    const size_t spare_rec = (nLs2 - nL - 1) * (size_t)n_resid;
    long long* base = nullptr;
    if ((st = m.get(&coeff, B * NG * H * nLs2 * C * r * sa)) != LOWRAM_OK ||
        (st = m.get(&summ, B * NG * H * nLs2 * r * 2)) != LOWRAM_OK ||
        (st = m.get(&rptr, U * (nLs2 + 1) * 4)) != LOWRAM_OK || (st = m.get(&base, (U + 1) * 8)) != LOWRAM_OK)
      return st;
    if (i8 && (st = m.get(&cscale, B * NG * H * nLs2 * C * 2)) != LOWRAM_OK) return st;
    if (c->cb.slot && (st = m.get(&slot, B * NG * H * nCs2 * 2)) != LOWRAM_OK) return st;
    e = rows2d(coeff, nLs2 * C * r * sa, c->cb.coeff, nLs * C * r * sa, nL * C * r * sa);
    if (e == cudaSuccess) e = rows2d(at(coeff, nL * C * r * sa), nLs2 * C * r * sa, dst.coeff, C * r * sa, C * r * sa);
    if (e == cudaSuccess && i8) {
      e = rows2d(cscale, nLs2 * C * 2, c->cb.coeff_scale, nLs * C * 2, nL * C * 2);
      if (e == cudaSuccess) e = rows2d(at(cscale, nL * C * 2), nLs2 * C * 2, dst.coeff_scale, C * 2, C * 2);
    }
    if (e == cudaSuccess) e = rows2d(summ, nLs2 * r * 2, c->cb.summary, nLs * r * 2, nL * r * 2);
    if (e == cudaSuccess) e = rows2d(at(summ, nL * r * 2), nLs2 * r * 2, dst.summary, r * 2, r * 2);
    if (e == cudaSuccess && slot) {
      e = rows2d(slot, nCs2 * 2, c->cb.slot, nCs * 2, nC * 2);
      if (e == cudaSuccess) e = launch_repack_slot((long long)(B * NG * H), (int)nCs2, (int)nC, (int)nL, slot, s);
    }
    if (e == cudaSuccess)
      e = launch_repack_scan((int)U, (int)nL, (int)nLs, (long long)spare_rec, c->cb.res_ptr, dst.res_ptr, base, err, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(&total, base + U, 8, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "re-lay the chunk arrays");
    if (total < 0 || total + kResPad >= (1LL << 31)) return inval("re-packed record count out of range");
    if ((st = m.get(&rpos, (size_t)total * 2)) != LOWRAM_OK ||
        (st = m.get(&rval, ((size_t)total + kResPad) * d * sa)) != LOWRAM_OK)
      return st;
    if (i8 && (st = m.get(&rscale, (size_t)total * 2)) != LOWRAM_OK) return st;
    // spare record rows are zero: the tensor-core kernel reads a fixed box of rows from a
    // chunk's first record and multiplies the rows past the chunk's records by zero
    e = cudaMemsetAsync(rval, 0, ((size_t)total + kResPad) * d * sa, s);
    if (e == cudaSuccess)
      e = launch_repack_records((int)U, (int)nL, (int)nLs, (int)nLs2, (int)(d * sa), c->cb.n_records, (long long)n_new,
                                c->cb.res_ptr, c->cb.res_pos, c->cb.res_val, c->cb.res_scale, dst.res_ptr, dst.res_pos,
                                dst.res_val, static_cast<const __half*>(dst.res_scale), base, rptr, rpos, rval, rscale,
                                err, s);
    if (e != cudaSuccess) return cuda_fail(e, "re-lay the residual records");
  }
  uint32_t word = 0, enc_word = 0;
  e = cudaMemcpyAsync(&word, err, 4, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(&enc_word, encode_error_word(ge, ws, true), 4, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "re-lay the residual records");
  word |= enc_word;
  // In place, only rows past the live ones were written so far: an error leaves the cache
  // as it was (its counts are unchanged).
  if (word & ERR_RES_PTR) {
    g_last_error = "the cache's CSR offsets are inconsistent: nothing re-packed";
    return LOWRAM_ECORRUPT;
  }
  if (word & ERR_TIMEOUT) {
    g_last_error = "the encoder gave up a bounded wait: nothing re-packed";
    return LOWRAM_ETIMEOUT;
  }
  if (!in_place && c->n_owned + 4 > (int)(sizeof(c->owned) / sizeof(c->owned[0])))
    return inval("internal: too many owned allocations");
  // 5. the tail drops its oldest chunk (the last step: the cache is unchanged until here)
  e = launch_tail_shift((int)B, (int)L, (int)H, T, C, (int)tail_row, const_cast<void*>(c->cb.tail_k),
                        const_cast<void*>(c->cb.tail_v), const_cast<int32_t*>(c->cb.tail_len), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "shift the tail");
  // 6. the new counts (and, after a re-lay, the new arrays)
  if (!in_place) {
    auto take = [&](const void* old_p, void* new_p) {
      m.release(new_p);
      swap_owned(c, old_p, new_p);
    };
    take(c->cb.coeff, coeff); c->cb.coeff = coeff;
    if (i8) { take(c->cb.coeff_scale, cscale); c->cb.coeff_scale = static_cast<const __half*>(cscale); }
    take(c->cb.summary, summ); c->cb.summary = summ;
    if (slot) { take(c->cb.slot, slot); c->cb.slot = slot; }
    take(c->cb.res_ptr, rptr); c->cb.res_ptr = rptr;
    take(c->cb.res_pos, rpos); c->cb.res_pos = rpos;
    take(c->cb.res_val, rval); c->cb.res_val = rval;
    if (i8) { take(c->cb.res_scale, rscale); c->cb.res_scale = rscale; }
    c->cb.n_records = total;
    c->nLs = (int)nLs2;
    c->nCs = (int)nCs2;
    c->canonical = true;
  }
  c->cfg.n_ctx += C;
  c->cfg.n_live += 1;
  c->nC += 1;
  c->nL += 1;
  c->generation += 1;
  c->last_repack_in_place = in_place;
  if (c->host_exec) {   // its kernels' geometry and pointers are those of the shorter cache
    cudaGraphExecDestroy(c->host_exec);
    c->host_exec = nullptr;
  }
  return LOWRAM_OK;
}

lowram_status lowram_cache_set_stage_events(lowram_cache* c, void* const* events) {
  if (!c) return inval("NULL cache");
  if (!events) {
    c->ev_on = false;
    return LOWRAM_OK;
  }
  for (int i = 0; i < 4; ++i) {
    if (!events[i]) return inval("NULL event");
    c->ev[i] = static_cast<cudaEvent_t>(events[i]);
  }
  c->ev_on = true;
  return LOWRAM_OK;
}

int32_t lowram_cache_last_launches(const lowram_cache* c) { return c ? c->last_launches : 0; }
int32_t lowram_cache_last_path(const lowram_cache* c) { return c ? c->last_path : -1; }

static lowram_status check_layers(const lowram_cache* c, int32_t layer0, int32_t n_layers) {
  if (!c) return inval("NULL cache");
  // written so that no sum can overflow: layer0 >= 0 first, then n_layers against the rest
  if (layer0 < 0 || n_layers < 1 || layer0 >= c->cfg.n_layers || n_layers > c->cfg.n_layers - layer0)
    return inval("layer range outside the cache");
  return LOWRAM_OK;
}

lowram_status lowram_select_chunks(lowram_cache* c, int32_t layer0, int32_t n_layers,
                                   const void* q, float* scores, int32_t* sel,
                                   lowram_stream stream) {
  lowram_status st = check_layers(c, layer0, n_layers);
  if (st != LOWRAM_OK) return st;
  if (!q) return inval("NULL q");
  Geom g = make_geom(c, layer0, n_layers, false);
  c->shard_l0 = -1;   // the scratch phase 1 of a sharded decode left is overwritten
  cudaError_t e = launch_select(g, c->cb, c->sc, c->cfg.dtype, q, scores, sel, 0, false,
                                reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "select kernel");
  return LOWRAM_OK;
}

lowram_status lowram_decode_attn(lowram_cache* c, int32_t layer0, int32_t n_layers,
                                 const void* q, void* out, int32_t* sel, int32_t path,
                                 lowram_stream stream) {
  lowram_status st = check_layers(c, layer0, n_layers);
  if (st != LOWRAM_OK) return st;
  if (!q || !out) return inval("NULL q or out");
  if (path < LOWRAM_PATH_AUTO || path > LOWRAM_PATH_TC) return inval("unknown path");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const bool tc_able = attend_tc_supported(make_geom(c, layer0, n_layers, true), c->cfg.dtype,
                                           c->cfg.store);
  bool tc = false;
  if (path == LOWRAM_PATH_TC) {
    if (!tc_able) {
      g_last_error = "the tensor-core path does not handle these shapes";
      return LOWRAM_EUNSUPPORTED;
    }
    tc = true;
  } else if (path == LOWRAM_PATH_AUTO) {
    tc = tc_able;
  }
  Geom g = make_geom(c, layer0, n_layers, tc);
  c->shard_l0 = -1;   // the scratch phase 1 of a sharded decode left is overwritten
  cudaError_t e;
  if (c->ev_on && (e = cudaEventRecord(c->ev[0], s)) != cudaSuccess) return cuda_fail(e, "event");
  const int tc_q_mode = tc ? (c->cfg.store == LOWRAM_STORE_INT8 ? 2 : 1) : 0;
  e = launch_select(g, c->cb, c->sc, c->cfg.dtype, q, nullptr, sel, tc_q_mode, true, s);
  if (e != cudaSuccess) return cuda_fail(e, "select kernel");
  if (c->ev_on && (e = cudaEventRecord(c->ev[1], s)) != cudaSuccess) return cuda_fail(e, "event");
  if (tc)
    e = launch_attend_tc(g, c->cb, c->sc, c->cfg.store, c->w1f_tc, c->n_sm, s);
  else
    e = launch_attend_simt(g, c->cb, c->sc, c->cfg.dtype, c->cfg.store, c->w1f_t, 0, s);
  if (e != cudaSuccess) return cuda_fail(e, "chunk attention kernel");
  if (c->ev_on && (e = cudaEventRecord(c->ev[2], s)) != cudaSuccess) return cuda_fail(e, "event");
  e = launch_combine(g, c->cb, c->sc, c->cfg.dtype, out, s);
  if (e != cudaSuccess) return cuda_fail(e, "combine kernel");
  if (c->ev_on && (e = cudaEventRecord(c->ev[3], s)) != cudaSuccess) return cuda_fail(e, "event");
  c->last_launches = 3;
  c->last_path = tc ? LOWRAM_PATH_TC : LOWRAM_PATH_SIMT;
  return LOWRAM_OK;
}

lowram_status lowram_decode_attn_host(lowram_cache* c, int32_t layer0, int32_t n_layers,
                                      const void* q_host, void* out_host, int32_t* sel_host,
                                      lowram_stream stream) {
  lowram_status st = check_layers(c, layer0, n_layers);
  if (st != LOWRAM_OK) return st;
  if (!q_host || !out_host) return inval("NULL q or out");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t qbytes = (size_t)n_layers * c->cfg.batch * c->cfg.n_q_heads * c->cfg.head_dim * c->s_dt;
  const size_t sbytes = (size_t)n_layers * c->cfg.batch * c->cfg.n_kv_heads * c->cfg.top_k * 4;
  cudaError_t e = cudaMemcpyAsync(c->q_stage, q_host, qbytes, cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return cuda_fail(e, "copy q to the device");
  int32_t* sel_dev = sel_host ? c->sel_stage : nullptr;
  bool replayed = false;
  if (!c->ev_on && !c->hg_off) {
    const bool same = c->host_exec && c->hg_layer0 == layer0 && c->hg_n == n_layers && c->hg_sel == (sel_dev != nullptr);
    if (!same) {
      if (c->host_exec) cudaGraphExecDestroy(c->host_exec);
      c->host_exec = nullptr;
      // capture on a stream of the cache's own (the legacy default stream cannot be captured)
      cudaGraph_t graph = nullptr;
      bool ok = c->cap_stream || cudaStreamCreateWithFlags(&c->cap_stream, cudaStreamNonBlocking) == cudaSuccess;
      ok = ok && cudaStreamBeginCapture(c->cap_stream, cudaStreamCaptureModeThreadLocal) == cudaSuccess;
      if (ok) {
        const lowram_status sc = lowram_decode_attn(c, layer0, n_layers, c->q_stage, c->out_stage, sel_dev,
                                                    LOWRAM_PATH_AUTO, reinterpret_cast<lowram_stream>(c->cap_stream));
        const cudaError_t ec = cudaStreamEndCapture(c->cap_stream, &graph);
        ok = sc == LOWRAM_OK && ec == cudaSuccess && graph &&
             cudaGraphInstantiate(&c->host_exec, graph, 0) == cudaSuccess;
        if (graph) cudaGraphDestroy(graph);
      }
      if (ok) {
        c->hg_layer0 = layer0;
        c->hg_n = n_layers;
        c->hg_sel = sel_dev != nullptr;
      } else {
        c->host_exec = nullptr;
        c->hg_off = true;
        cudaGetLastError();   // clear a capture error; the eager call below reports its own
      }
    }
    if (c->host_exec) {
      e = cudaGraphLaunch(c->host_exec, s);
      if (e != cudaSuccess) return cuda_fail(e, "decode graph launch");
      replayed = true;
    }
  }
  if (!replayed) {
    st = lowram_decode_attn(c, layer0, n_layers, c->q_stage, c->out_stage, sel_dev, LOWRAM_PATH_AUTO, stream);
    if (st != LOWRAM_OK) return st;
  }
  e = cudaMemcpyAsync(out_host, c->out_stage, qbytes, cudaMemcpyDeviceToHost, s);
  if (e != cudaSuccess) return cuda_fail(e, "copy out to the host");
  if (sel_host) {
    e = cudaMemcpyAsync(sel_host, c->sel_stage, sbytes, cudaMemcpyDeviceToHost, s);
    if (e != cudaSuccess) return cuda_fail(e, "copy sel to the host");
  }
  e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  return LOWRAM_OK;
}

lowram_status lowram_cache_validate(lowram_cache* c, lowram_stream stream) {
  if (!c) return inval("NULL cache");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  Geom g = make_geom(c, 0, c->cfg.n_layers, false);
  cudaError_t e = launch_validate(g, c->cb, c->sc.err, s);
  if (e != cudaSuccess) return cuda_fail(e, "validate kernel");
  uint32_t word = 0;
  e = cudaMemcpyAsync(&word, c->sc.err, 4, cudaMemcpyDeviceToHost, s);
  if (e != cudaSuccess) return cuda_fail(e, "read error word");
  e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  e = cudaMemsetAsync(c->sc.err, 0, 4, s);
  if (e != cudaSuccess) return cuda_fail(e, "clear error word");
  e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  if (word & (ERR_SLOT | ERR_RES_PTR | ERR_RES_POS | ERR_TAIL_LEN | ERR_SELECT)) {
    char buf[96];
    std::snprintf(buf, sizeof buf, "cache tables inconsistent (error word 0x%x)", word);
    g_last_error = buf;
    return LOWRAM_ECORRUPT;
  }
  if (word & ERR_TIMEOUT) {
    g_last_error = "a kernel gave up a bounded wait";
    return LOWRAM_ETIMEOUT;
  }
  if (word & ERR_TAIL_FULL) {
    g_last_error = "an append found a full tail: that sequence's token was dropped";
    return LOWRAM_EINVAL;
  }
  return LOWRAM_OK;
}

// ------------------------------------------------------------- context-sharded decode

lowram_status lowram_shard_candidates(lowram_cache* c, int32_t layer0, int32_t n_layers, const void* q,
                                      int32_t chunk_offset, float* cand_score, int32_t* cand_id,
                                      lowram_stream stream) {
  lowram_status st = check_layers(c, layer0, n_layers);
  if (st != LOWRAM_OK) return st;
  if (!q || !cand_score || !cand_id) return inval("NULL q or candidate output");
  if (chunk_offset < 0) return inval("chunk_offset must be >= 0");
  Geom g = make_geom(c, layer0, n_layers, true);
  if (!attend_tc_supported(g, c->cfg.dtype, c->cfg.store)) {
    g_last_error = "context-sharded decode runs on the tensor-core kernel's shapes only";
    return LOWRAM_EUNSUPPORTED;
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int tc_q_mode = c->cfg.store == LOWRAM_STORE_INT8 ? 2 : 1;
  cudaError_t e = launch_select(g, c->cb, c->sc, c->cfg.dtype, q, nullptr, nullptr, tc_q_mode, true, s,
                                SelCand{cand_score, cand_id, chunk_offset});
  if (e != cudaSuccess) return cuda_fail(e, "select kernel");
  c->shard_l0 = layer0;
  c->shard_n = n_layers;
  c->last_launches = 1;
  return LOWRAM_OK;
}

lowram_status lowram_shard_partial(lowram_cache* c, int32_t layer0, int32_t n_layers, int32_t chunk_offset,
                                   int32_t n_shards, const float* cand_score, const int32_t* cand_id,
                                   float* partial, int32_t* sel, lowram_stream stream) {
  lowram_status st = check_layers(c, layer0, n_layers);
  if (st != LOWRAM_OK) return st;
  if (!cand_score || !cand_id || !partial) return inval("NULL candidates or partial output");
  if (chunk_offset < 0) return inval("chunk_offset must be >= 0");
  if (n_shards < 1 || (long long)n_shards * c->cfg.top_k > 1024)
    return inval("n_shards must be >= 1 with n_shards * top_k <= 1024");
  if (layer0 != c->shard_l0 || n_layers != c->shard_n)
    return inval("lowram_shard_partial must follow lowram_shard_candidates for the same layers on this cache");
  Geom g = make_geom(c, layer0, n_layers, true);
  if (!attend_tc_supported(g, c->cfg.dtype, c->cfg.store)) {
    g_last_error = "context-sharded decode runs on the tensor-core kernel's shapes only";
    return LOWRAM_EUNSUPPORTED;
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  Scratch sc = c->sc;
  sc.tile_unit = c->t_unit;
  sc.tile_slot = c->t_slot;
  sc.tile_ptr = c->t_ptr;
  sc.tile_total = c->t_total;
  sc.unit_ntile = c->t_cnt;
  cudaError_t e = launch_shard_select(g, c->cb, sc, cand_score, cand_id, n_shards, chunk_offset, sel, s);
  if (e != cudaSuccess) return cuda_fail(e, "shard selection kernels");
  e = launch_attend_tc(g, c->cb, sc, c->cfg.store, c->w1f_tc, c->n_sm, s);
  if (e != cudaSuccess) return cuda_fail(e, "chunk attention kernel");
  e = launch_combine_partial(g, c->cb, sc, c->cfg.dtype, partial, s);
  if (e != cudaSuccess) return cuda_fail(e, "partial combine kernel");
  c->last_launches = 4;
  c->last_path = LOWRAM_PATH_TC;
  return LOWRAM_OK;
}

lowram_status lowram_merge_partials(int32_t n_parts, int64_t n_rows, int32_t head_dim, const float* partials,
                                    int32_t out_dtype, void* out, lowram_stream stream) {
  if (n_parts < 1 || n_rows < 0 || n_rows >= (1LL << 31) || head_dim < 1 || head_dim > kMaxD)
    return inval("n_parts >= 1, 0 <= n_rows < 2^31 and 1 <= head_dim <= 256 are required");
  if (out_dtype != LOWRAM_F32 && out_dtype != LOWRAM_BF16) return inval("unknown output dtype");
  if (n_rows > 0 && (!partials || !out)) return inval("NULL partials or out");
  cudaError_t e = launch_merge_partials(n_parts, n_rows, head_dim, partials, out_dtype, out,
                                        reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "merge kernel");
  return LOWRAM_OK;
}

// ------------------------------------------------------------- reuse of rebuilt chunks

void lowram_reuse_destroy(lowram_reuse* r) {
  if (!r) return;
  cudaDeviceSynchronize();
  for (int i = 0; i < r->n_mem; ++i) cudaFree(r->mem[i]);
  delete r;
}

lowram_status lowram_reuse_create(lowram_cache* c, int32_t capacity, int32_t fill_cap, lowram_reuse** out,
                                  lowram_stream stream) {
  if (out) *out = nullptr;
  if (!c || !out) return inval("NULL cache or output");
  // capacity <= 2^30 keeps the ring arithmetic (position + fill index < 2 * capacity) in int32
  if (capacity < 1 || capacity > (1 << 30) || fill_cap < 0 || fill_cap > capacity)
    return inval("need 1 <= capacity <= 2^30 and 0 <= fill_cap <= capacity");
  Geom g = make_geom(c, 0, c->cfg.n_layers, true);
  if (!reuse_supported(g, c->cfg.dtype, c->cfg.store) || c->cfg.top_k > 32) {
    g_last_error = "the reuse store takes bf16 native stores, head_dim 128, mlp_hidden 256, rank 64 or 128, "
                   "chunk 128, 4 or 8 query heads per KV head and top_k <= 32";
    return LOWRAM_EUNSUPPORTED;
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  lowram_reuse* r = new lowram_reuse();
  std::memset(r, 0, sizeof(*r));
  r->cache = c;
  r->generation = c->generation;
  const size_t B = c->cfg.batch, L = c->cfg.n_layers, H = c->cfg.n_kv_heads, d = c->cfg.head_dim;
  const size_t C = c->cfg.chunk, h = c->cfg.mlp_hidden, k = c->cfg.top_k, Umax = B * L * H;
  const size_t table_n = Umax * (size_t)c->nLs;
  const size_t tail_stride = (size_t)g.tail_stride;
  struct Piece { void** p; size_t bytes; };
  Piece pieces[] = {
      {reinterpret_cast<void**>(&r->d.entries), (size_t)capacity * C * d * 2},
      {reinterpret_cast<void**>(&r->d.table), table_n * 4},
      {reinterpret_cast<void**>(&r->d.owner), (size_t)capacity * 8},
      {reinterpret_cast<void**>(&r->d.ring), 16},
      {reinterpret_cast<void**>(&r->d.counters), 32},
      {reinterpret_cast<void**>(&r->d.hit_entry), Umax * k * 4},
      {reinterpret_cast<void**>(&r->d.hit_slot), Umax * k * 4},
      {reinterpret_cast<void**>(&r->d.hit_n), Umax * 4},
      {reinterpret_cast<void**>(&r->d.hit_part), Umax * tail_stride * 4},
      {const_cast<void**>(reinterpret_cast<const void**>(&r->d.w2h)), L * H * d * h * 2},
  };
  for (Piece& pc : pieces) {
    cudaError_t e = device_malloc(pc.p, pc.bytes ? pc.bytes : 16);
    if (e != cudaSuccess) {
      lowram_reuse_destroy(r);
      g_last_error = std::string("cudaMalloc: ") + cudaGetErrorString(e);
      return LOWRAM_ENOMEM;
    }
    r->mem[r->n_mem++] = *pc.p;
  }
  r->d.E = capacity;
  r->d.fill_cap = fill_cap;
  r->d.table_stride = c->nLs;
  cudaError_t e = cudaMemsetAsync(r->d.table, 0xff, table_n * 4, s);   // -1: no entry
  if (e == cudaSuccess) e = cudaMemsetAsync(r->d.owner, 0xff, (size_t)capacity * 8, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(r->d.ring, 0, 16, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(r->d.counters, 0, 32, s);
  if (e == cudaSuccess) e = launch_to_half(static_cast<const __nv_bfloat16*>(c->cb.w2), const_cast<__half*>(r->d.w2h),
                                           L * H * d * h, s);
  if (e != cudaSuccess) {
    lowram_reuse_destroy(r);
    return cuda_fail(e, "initialise the reuse store");
  }
  *out = r;
  return LOWRAM_OK;
}

lowram_status lowram_decode_attn_reuse(lowram_reuse* r, int32_t layer0, int32_t n_layers, const void* q, void* out,
                                       int32_t* sel, lowram_stream stream) {
  if (!r) return inval("NULL store");
  lowram_cache* c = r->cache;
  lowram_status st = check_layers(c, layer0, n_layers);
  if (st != LOWRAM_OK) return st;
  if (!q || !out) return inval("NULL q or out");
  if (r->generation != c->generation) return inval("the cache was re-packed after the store was made: make a new one");
  Geom g = make_geom(c, layer0, n_layers, true);
  if (!attend_tc_supported(g, c->cfg.dtype, c->cfg.store) || !reuse_supported(g, c->cfg.dtype, c->cfg.store)) {
    g_last_error = "these shapes have no reuse path";
    return LOWRAM_EUNSUPPORTED;
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  c->shard_l0 = -1;
  cudaError_t e = launch_select(g, c->cb, c->sc, c->cfg.dtype, q, nullptr, sel, 1, true, s);
  if (e != cudaSuccess) return cuda_fail(e, "select kernel");
  Scratch sc = c->sc;
  sc.tile_unit = c->t_unit;
  sc.tile_slot = c->t_slot;
  sc.tile_ptr = c->t_ptr;
  sc.tile_total = c->t_total;
  sc.unit_ntile = c->t_cnt;
  if ((e = launch_reuse(g, c->cb, sc, r->d, c->w1f_tc, c->n_sm, s, 0)) != cudaSuccess) return cuda_fail(e, "reuse plan");
  if ((e = launch_attend_tc(g, c->cb, sc, c->cfg.store, c->w1f_tc, c->n_sm, s)) != cudaSuccess)
    return cuda_fail(e, "chunk attention kernel");
  if ((e = launch_reuse(g, c->cb, sc, r->d, c->w1f_tc, c->n_sm, s, 1)) != cudaSuccess) return cuda_fail(e, "reuse hits");
  if ((e = launch_combine_list(g, c->cb, sc, r->d.hit_part, out, s)) != cudaSuccess) return cuda_fail(e, "combine kernel");
  if ((e = launch_reuse(g, c->cb, sc, r->d, c->w1f_tc, c->n_sm, s, 2)) != cudaSuccess) return cuda_fail(e, "reuse fills");
  c->last_launches = 8;
  c->last_path = LOWRAM_PATH_TC;
  return LOWRAM_OK;
}

lowram_status lowram_reuse_counts_get(lowram_reuse* r, lowram_reuse_counts* out, lowram_stream stream) {
  if (!r || !out) return inval("NULL store or output");
  unsigned long long v[3];
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(v, r->d.counters, sizeof v, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "read the reuse counters");
  out->hits = v[0];
  out->misses = v[1];
  out->fills = v[2];
  return LOWRAM_OK;
}

lowram_status lowram_reuse_view(const lowram_reuse* r, const int32_t** table, const int64_t** owner,
                                const void** entries, int64_t* table_stride) {
  if (!r || !table || !owner || !entries || !table_stride) return inval("NULL store or output");
  *table = r->d.table;
  *owner = reinterpret_cast<const int64_t*>(r->d.owner);
  *entries = r->d.entries;
  *table_stride = r->d.table_stride;
  return LOWRAM_OK;
}

lowram_status lowram_debug_set_wait_limit(lowram_cache* c, int64_t cycles) {
  if (!c) return inval("NULL cache");
  c->wait_limit = cycles > 0 ? (long long)cycles : kDefaultWaitCycles;
  if (c->host_exec) {   // the captured graph holds the old limit
    cudaGraphExecDestroy(c->host_exec);
    c->host_exec = nullptr;
  }
  return LOWRAM_OK;
}

void lowram_debug_fail_alloc(int32_t after) { g_fail_after.store(after < 0 ? -1 : after); }

}  // extern "C"
