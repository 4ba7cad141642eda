// Decode-time attention without any device allocation.
//
// Some callers cannot call cudaMalloc on their decode path: an inference engine that
// reserves all device memory for its own pool at start-up, code that must not allocate
// after initialisation (latency-critical or certified runtimes), or a thread that is
// capturing a CUDA graph in a mode that forbids allocation calls.  For them,
// lowram_decode_attn_static runs the same CUDA-core decode kernels as
// lowram_decode_attn, but reads the compressed cache straight from the caller's arrays
// (no cache object, no copies) and keeps every piece of scratch -- the folded predictor
// weights of the requested layers, the projected queries, the selection, the split
// partials and the error word -- in one file-scope static device array of
// kStaticScratchBytes.  Each GPU that loads the library holds that array until the
// process exits.
#include <mutex>
#include <string>

#include "lowram_internal.cuh"

namespace lowram {
void set_last_error(const char* msg);
}

using namespace lowram;

namespace {

constexpr size_t kStaticScratchBytes = size_t(16) << 20;   // 16 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

std::mutex g_addr_mu;
void* g_addr[kMaxDevices] = {};

size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

lowram_status fail_cuda(cudaError_t e, const char* where) {
  std::string m = std::string(where) + ": " + cudaGetErrorString(e);
  set_last_error(m.c_str());
  return LOWRAM_ECUDA;
}

lowram_status fail_inval(const std::string& m) {
  set_last_error(m.c_str());
  return LOWRAM_EINVAL;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Device address of the static array on the current device (looked up once per device).
lowram_status static_base(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail_cuda(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail_inval("device index above 63");
  std::lock_guard<std::mutex> lock(g_addr_mu);
  if (!g_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return fail_cuda(e, "cudaGetSymbolAddress");
    g_addr[dev] = p;
  }
  *out = g_addr[dev];
  return LOWRAM_OK;
}

}  // namespace

extern "C" lowram_status lowram_decode_attn_static(const lowram_config* cfg,
                                                   const lowram_cache_src* src, int32_t layer0,
                                                   int32_t n_layers, const void* q, void* out,
                                                   int32_t* sel, lowram_stream stream) {
  lowram_bytes nb;
  lowram_status st = lowram_config_bytes(cfg, src ? src->n_records : 0, 0, &nb);  // shape checks
  if (st != LOWRAM_OK) return st;
  if (!src || !q || !out) return fail_inval("NULL src, q or out");
  if (layer0 < 0 || n_layers < 1 || layer0 >= cfg->n_layers || n_layers > cfg->n_layers - layer0)
    return fail_inval("layer range outside the cache");
  const bool i8 = cfg->store == LOWRAM_STORE_INT8;
  const int nC = cfg->n_ctx / cfg->chunk;
  const bool evict = cfg->n_live < nC;
  const void* need[] = {src->coeff, src->basis, src->w1, src->w2, src->summary, src->res_ptr,
                        src->tail_k, src->tail_v, src->tail_len};
  for (const void* p : need)
    if (!p || !aligned16(p)) return fail_inval("a required source pointer is NULL or not 16-byte aligned");
  if (src->n_records < 0 || src->n_records >= (1LL << 31)) return fail_inval("n_records out of range");
  if (src->n_records > 0 && (!src->res_pos || !src->res_val)) return fail_inval("residual arrays missing");
  if (i8 && (!src->coeff_scale || (src->n_records > 0 && !src->res_scale)))
    return fail_inval("int8 store needs coeff_scale and res_scale");
  if (evict && !src->slot) return fail_inval("eviction needs a slot map");

  int dev = 0, n_sm = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail_cuda(e, "cudaGetDevice");
  e = cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return fail_cuda(e, "cudaDeviceGetAttribute");

  Geom g;
  g.B = cfg->batch; g.L = cfg->n_layers; g.G = cfg->group; g.Hkv = cfg->n_kv_heads;
  g.Hq = cfg->n_q_heads; g.g = g.Hq / g.Hkv; g.d = cfg->head_dim; g.r = cfg->rank;
  g.h = cfg->mlp_hidden; g.N = cfg->n_ctx; g.C = cfg->chunk; g.nC = nC; g.nL = cfg->n_live;
  g.nLs = g.nL; g.nCs = g.nC;
  g.k = cfg->top_k; g.T = cfg->tail_cap; g.layer0 = layer0; g.n_layers = n_layers;
  g.U = n_layers * g.Hkv * g.B;
  const long long total = (long long)g.U * g.k;
  g.P = (int)(total < 4LL * n_sm ? total : 4LL * n_sm);
  g.rec_stride = (2 * g.g + g.g * g.h + g.g * g.d + 3) & ~3;
  g.tail_stride = (2 * g.g + g.g * g.d + 3) & ~3;
  g.max_rec = max_records_per_unit(total, g.P, g.k);
  g.qk_scale_log2 = 1.4426950408889634f / sqrtf((float)g.d);
  g.wait_cycles = kDefaultWaitCycles;

  // carve the static array: error word, folded W1' of the requested layers, projected
  // queries, selection, split partials, tail partials
  const size_t lw = (size_t)n_layers * g.Hkv * g.r * g.h;
  size_t off = 0;
  const size_t o_err = off;  off += 256;
  const size_t o_w1f = off;  off += round256(lw * 4);
  const size_t o_qt = off;   off += round256((size_t)g.U * g.g * g.r * 4);
  const size_t o_ss = off;   off += round256((size_t)g.U * g.k * 4);
  const size_t o_si = off;   off += round256((size_t)g.U * g.k * 4);
  const size_t o_part = off; off += round256(((size_t)g.U + g.P) * g.rec_stride * 4);
  const size_t o_tail = off; off += round256((size_t)g.U * g.tail_stride * 4);
  if (off > kStaticScratchBytes) {
    return fail_inval("lowram_decode_attn_static needs " + std::to_string(off) +
                      " bytes of scratch for this call, above the static maximum of " +
                      std::to_string(kStaticScratchBytes) + " bytes: decode fewer layers per call");
  }
  void* base = nullptr;
  if ((st = static_base(&base)) != LOWRAM_OK) return st;
  unsigned char* sb = static_cast<unsigned char*>(base);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

  Scratch sc{};
  sc.err = reinterpret_cast<uint32_t*>(sb + o_err);
  sc.qt = reinterpret_cast<float*>(sb + o_qt);
  sc.qt_tc = nullptr;
  sc.sel_slot = reinterpret_cast<int32_t*>(sb + o_ss);
  sc.sel_id = reinterpret_cast<int32_t*>(sb + o_si);
  sc.part = reinterpret_cast<float*>(sb + o_part);
  sc.tail_part = reinterpret_cast<float*>(sb + o_tail);
  // the array keeps the previous call's contents: the error word must start at zero
  e = cudaMemsetAsync(sc.err, 0, 4, s);
  if (e != cudaSuccess) return fail_cuda(e, "cudaMemsetAsync");

  CacheBuffers cb;
  cb.coeff = src->coeff;
  cb.coeff_scale = static_cast<const __half*>(src->coeff_scale);
  cb.basis = src->basis; cb.w1 = src->w1; cb.w2 = src->w2; cb.summary = src->summary;
  cb.slot = evict ? src->slot : nullptr;
  cb.res_ptr = src->res_ptr; cb.res_pos = src->res_pos; cb.res_val = src->res_val;
  cb.res_scale = static_cast<const __half*>(src->res_scale);
  cb.tail_k = src->tail_k; cb.tail_v = src->tail_v; cb.tail_len = src->tail_len;
  cb.n_records = src->n_records;

  // fold W1' = W1 B_l^T for layers [layer0, layer0 + n_layers) only
  const size_t es = cfg->dtype == LOWRAM_F32 ? 4 : 2;
  CacheBuffers cbf = cb;
  cbf.w1 = static_cast<const unsigned char*>(src->w1) + (size_t)layer0 * g.Hkv * g.h * g.d * es;
  cbf.basis = static_cast<const unsigned char*>(src->basis) + (size_t)layer0 * g.Hkv * g.r * g.d * es;
  Geom gf = g;
  gf.L = n_layers;
  float* w1f = reinterpret_cast<float*>(sb + o_w1f);
  e = launch_fold(gf, cbf, cfg->dtype, cfg->store, w1f, nullptr, s);
  if (e != cudaSuccess) return fail_cuda(e, "fold kernel");

  e = launch_select(g, cb, sc, cfg->dtype, q, nullptr, sel, 0, true, s);
  if (e != cudaSuccess) return fail_cuda(e, "select kernel");
  // w1f holds layers [layer0, layer0 + n_layers): the kernel indexes it from layer0
  e = launch_attend_simt(g, cb, sc, cfg->dtype, cfg->store, w1f, layer0, s);
  if (e != cudaSuccess) return fail_cuda(e, "chunk attention kernel");
  e = launch_combine(g, cb, sc, cfg->dtype, out, s);
  if (e != cudaSuccess) return fail_cuda(e, "combine kernel");
  return LOWRAM_OK;
}
