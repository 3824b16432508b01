// libvsa.cu -- the C ABI (declared in include/vsa.h): argument checks, tile
// geometry, TMA descriptor encoding and kernel launches.  The only translation
// unit of libvsa.so; the kernels live in the headers it includes.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <atomic>
#include <mutex>

#include "vsa.h"
#include "attn_kernel.cuh"
#include "select_kernels.cuh"
#include "tma_encode.cuh"
#include "vsa_geometry.cuh"

namespace vsa {

__device__ unsigned int g_device_error = 0u;

constexpr int kMaxTiles = 1536;          // score rows of one CTA must fit in shared memory
constexpr int kMaxDevices = 64;
constexpr int kMaxSmemPerBlock = 232448;  // opt-in dynamic shared memory per CTA on sm_100

// -------------------------------------------------------------- validation
// One side's grid and tile: positive extents, power-of-two tile extents with
// a supported volume, tile counts and index ranges within the kernels' limits.
static int side_geom(const vsa_shape* s, int T, int Hh, int W, int tt, int th, int tw, Geom* g) {
  if (T <= 0 || Hh <= 0 || W <= 0 || tt <= 0 || th <= 0 || tw <= 0) return VSA_ERR_INVALID_ARG;
  const int lt = ilog2_exact(tt), ly = ilog2_exact(th), lx = ilog2_exact(tw);
  if (lt < 0 || ly < 0 || lx < 0) return VSA_ERR_UNSUPPORTED;
  if (tt > 256 || th > 256 || tw > 256) return VSA_ERR_UNSUPPORTED;
  const int vol = tt * th * tw;
  if (vol != 64 && vol != 128 && vol != 256) return VSA_ERR_UNSUPPORTED;
  if (vol == 256 && tt < 2) return VSA_ERR_UNSUPPORTED;
  g->B = s->B; g->H = s->H; g->T = T; g->Hh = Hh; g->W = W; g->d = s->d;
  g->tt = tt; g->th = th; g->tw = tw;
  g->lg_tt = lt; g->lg_th = ly; g->lg_tw = lx;
  g->vol = vol;
  g->f16 = s->dtype == VSA_DTYPE_F16 ? 1 : 0;
  g->layout = s->layout;
  g->prefix = 0;
  g->nTt = ceil_div(T, tt);
  g->nTy = ceil_div(Hh, th);
  g->nTx = ceil_div(W, tw);
  const long long nT = 1ll * g->nTt * g->nTy * g->nTx;
  const long long N = 1ll * T * Hh * W;
  const long long BH = 1ll * s->B * s->H;
  // grid-dimension and index limits of the kernels
  if (nT > kMaxTiles || BH > 65535 || BH * nT > 0x7fffffffll || N * s->d * BH > (1ll << 40) ||
      1ll * s->B * T > 0x7fffffffll)
    return VSA_ERR_TOO_LARGE;
  g->nT = static_cast<int>(nT);
  return VSA_OK;
}

// Query-side and key/value-side geometry of a shape (the key/value grid and
// tile default to the query's when left zero).
static int make_geoms(const vsa_shape* s, Geom* gq, Geom* gk) {
  if (s == nullptr) return VSA_ERR_INVALID_ARG;
  if (s->B <= 0 || s->H <= 0 || s->d <= 0) return VSA_ERR_INVALID_ARG;
  if (s->d != 64 && s->d != 128) return VSA_ERR_UNSUPPORTED;
  if (s->dtype != VSA_DTYPE_BF16 && s->dtype != VSA_DTYPE_F16) return VSA_ERR_UNSUPPORTED;
  if (s->layout != VSA_LAYOUT_BHND && s->layout != VSA_LAYOUT_BNHD) return VSA_ERR_UNSUPPORTED;
  int rc = side_geom(s, s->T, s->Hh, s->W, s->tt, s->th, s->tw, gq);
  if (rc != VSA_OK) return rc;
  const bool kgrid = s->Tk != 0 || s->Hk != 0 || s->Wk != 0;
  const bool ktile = s->tk != 0 || s->hk != 0 || s->wk != 0;
  rc = side_geom(s, kgrid ? s->Tk : s->T, kgrid ? s->Hk : s->Hh, kgrid ? s->Wk : s->W, ktile ? s->tk : s->tt,
                 ktile ? s->hk : s->th, ktile ? s->wk : s->tw, gk);
  if (rc != VSA_OK) return rc;
  if (gq->vol != gk->vol) return VSA_ERR_UNSUPPORTED;
  if (s->prefix_tiles < 0 || s->prefix_tiles > gk->nT) return VSA_ERR_INVALID_ARG;
  gk->prefix = s->prefix_tiles;
  return VSA_OK;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static int check_arch() {
  static int cached[kMaxDevices];          // 0 unknown, 1 ok, 2 bad
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return VSA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return VSA_ERR_ARCH;
  if (cached[dev] == 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return VSA_ERR_CUDA;
    cached[dev] = (major == 10 && minor == 0) ? 1 : 2;
  }
  return cached[dev] == 1 ? VSA_OK : VSA_ERR_ARCH;
}

// Device addresses of this library's __device__ arrays, looked up with
// cudaGetSymbolAddress once per device and context and cached: a symbol's
// address is fixed for the life of the context that loaded the module, and a
// new context (after cudaDeviceReset, say) loads it again elsewhere, so the
// cache is keyed by the context's process-unique id.  The driver calls are
// reached through the runtime's entry-point query (no link against libcuda).
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

static bool current_ctx_id(unsigned long long* id) {
  static CtxGetCurrentFn get_cur = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_cur = reinterpret_cast<CtxGetCurrentFn>(p);
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  CUcontext ctx = nullptr;
  if (get_cur == nullptr || get_id == nullptr || get_cur(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

struct SymbolCache {
  void* ptr[kMaxDevices] = {};
  unsigned long long ctx[kMaxDevices] = {};
  std::mutex mu;
};

// Address of `symbol` on the current device (its context is created by the
// lookup if the runtime has not made one yet).
static int symbol_address(const void* symbol, SymbolCache& c, void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return VSA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return VSA_ERR_ARCH;
  std::lock_guard<std::mutex> lock(c.mu);
  unsigned long long id = 0;
  if (c.ptr[dev] == nullptr || !current_ctx_id(&id) || id != c.ctx[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, symbol) != cudaSuccess || p == nullptr) return VSA_ERR_CUDA;
    if (!current_ctx_id(&id)) return VSA_ERR_CUDA;
    c.ptr[dev] = p;
    c.ctx[dev] = id;
  }
  *out = c.ptr[dev];
  return VSA_OK;
}

static unsigned int* device_error_ptr() {
  static SymbolCache cache;
  void* p = nullptr;
  return symbol_address(&g_device_error, cache, &p) == VSA_OK ? static_cast<unsigned int*>(p) : nullptr;
}

// Score + top-k grid, launched as a programmatic dependent of the pooling
// grid: its CTAs may start while pooling drains; griddepcontrol.wait holds
// them until the pooled means are complete.  Heads of kNarrowMaxTiles + 1 ..
// kWideLongMaxTiles key tiles take the wide kernel (32 query tiles per CTA;
// a 2-deep ring past kWideMaxTiles); smaller heads (little score work, more
// CTAs) and larger ones (key rows that would not fit beside the wide ring)
// take the narrow kernel (16).
template <int D, int STAGES, int KEYS>
static int launch_score_wide(const Geom& gq, const Geom& gk, int topk, int32_t* idx, const float* means,
                             const cudaLaunchAttribute* attr, cudaStream_t st) {
  const size_t smem = score_smem_bytes<D, STAGES, KEYS>(gk);
  if (cudaFuncSetAttribute(score_topk_kernel<D, STAGES, KEYS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return VSA_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ceil_div(gq.nT, kWideRows), gq.B * gq.H);
  cfg.blockDim = dim3(kWideThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = const_cast<cudaLaunchAttribute*>(attr);
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, score_topk_kernel<D, STAGES, KEYS>, gq, gk, means, topk, idx) == cudaSuccess
             ? VSA_OK
             : VSA_ERR_CUDA;
}

template <int D, int KEYS, int STAGES>
static int launch_score_narrow(const Geom& gq, const Geom& gk, int topk, int32_t* idx, const float* means,
                               const cudaLaunchAttribute* attr, cudaStream_t st) {
  const size_t smem = score_narrow_smem_bytes<D, KEYS, STAGES>(gk);
  if (cudaFuncSetAttribute(score_topk_narrow_kernel<D, KEYS, STAGES>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return VSA_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ceil_div(gq.nT, kNarrowRows), gq.B * gq.H);
  cfg.blockDim = dim3(kNarrowThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = const_cast<cudaLaunchAttribute*>(attr);
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, score_topk_narrow_kernel<D, KEYS, STAGES>, gq, gk, means, topk, idx) ==
                 cudaSuccess
             ? VSA_OK
             : VSA_ERR_CUDA;
}

template <int D>
static int launch_score(const Geom& gq, const Geom& gk, int topk, int32_t* idx, const float* means,
                        cudaStream_t st) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  if (gk.nT > kNarrowMaxTiles && gk.nT <= kWideKeys)
    return launch_score_wide<D, kWideStages, kWideKeys>(gq, gk, topk, idx, means, attr, st);
  if (gk.nT > kWideKeys && gk.nT <= kWideMaxTiles)          // one pass, 12 math warps, 2-deep ring
    return launch_score_wide<D, 2, kWideKeysOne>(gq, gk, topk, idx, means, attr, st);
  if (gk.nT > kWideMaxTiles && gk.nT <= kWideLongMaxTiles)
    return launch_score_wide<D, kWideStagesLong, kWideKeys>(gq, gk, topk, idx, means, attr, st);
  return gk.nT <= kShortKeys ? launch_score_narrow<D, kShortKeys, kShortStages>(gq, gk, topk, idx, means, attr, st)
                             : launch_score_narrow<D, kNarrowKeys, kNarrowStages>(gq, gk, topk, idx, means, attr, st);
}

// Tile-level attention of the pooled coarse branch: QT query tiles per warp,
// MAXJ key tiles per lane (see coarse_kernel).
template <int D, int MAXJ, int QT>
static int launch_coarse_j(const Geom& gq, const Geom& gk, const float* means, float scale_log2, float* out,
                           cudaStream_t st) {
  const size_t smem = coarse_smem_bytes<D>(gk, QT);
  if (cudaFuncSetAttribute(coarse_kernel<D, MAXJ, QT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return VSA_ERR_CUDA;
  coarse_kernel<D, MAXJ, QT><<<dim3(ceil_div(gq.nT, kCoarseWarps * QT), gq.B * gq.H), kCoarseWarps * 32, smem, st>>>(
      gq, gk, means, scale_log2, out);
  return cudaGetLastError() == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

template <int D>
static int launch_coarse(const Geom& gq, const Geom& gk, const float* means, float scale_log2, float* out,
                         cudaStream_t st) {
  if (gk.nT <= 256) return launch_coarse_j<D, 8, 4>(gq, gk, means, scale_log2, out, st);
  if (gk.nT <= 512) return launch_coarse_j<D, 16, 4>(gq, gk, means, scale_log2, out, st);
  if (gk.nT <= 768) return launch_coarse_j<D, 24, 4>(gq, gk, means, scale_log2, out, st);
  if (gk.nT <= 1024) return launch_coarse_j<D, 32, 2>(gq, gk, means, scale_log2, out, st);
  return launch_coarse_j<D, 48, 2>(gq, gk, means, scale_log2, out, st);
}

// Pooling (Q and K; with v != nullptr also V for the coarse branch), then
// scores + top-k; with v, then the coarse branch's tile-level attention.
template <int D, bool F16>
static int launch_select(const Geom& gq, const Geom& gk, const void* q, const void* k, const void* v, int topk,
                         int32_t* idx, void* ws, float scale_log2, float* coarse, cudaStream_t st) {
  CUtensorMap mq, mk, mv;
  int rc;
  if ((rc = encode_qkv_map(&mq, q, gq, gq.tt, F16)) != VSA_OK || (rc = encode_qkv_map(&mk, k, gk, gk.tt, F16)) != VSA_OK)
    return rc;
  if (v != nullptr && (rc = encode_qkv_map(&mv, v, gk, gk.tt, F16)) != VSA_OK) return rc;
  unsigned int* err = device_error_ptr();
  if (err == nullptr) return VSA_ERR_CUDA;
  float* means = static_cast<float*>(ws);
  const size_t psmem = pool_smem_bytes<D>(gq);
  if (cudaFuncSetAttribute(pool_kernel<D, F16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(psmem)) != cudaSuccess)
    return VSA_ERR_CUDA;
  pool_kernel<D, F16><<<dim3(max(gq.nT, gk.nT), gq.B * gq.H, v != nullptr ? 3 : 2), kPoolThreads, psmem, st>>>(
      mq, mk, v != nullptr ? mv : mk, gq, gk, means, err);
  if (cudaGetLastError() != cudaSuccess) return VSA_ERR_CUDA;
  if ((rc = launch_score<D>(gq, gk, topk, idx, means, st)) != VSA_OK) return rc;
  return v != nullptr ? launch_coarse<D>(gq, gk, means, scale_log2, coarse, st) : VSA_OK;
}

template <int D, int MODE, bool F16, bool SAME, bool BNHD>
static int launch_attn(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mo,
                       const AttnArgs& a, cudaStream_t st) {
  const int smem = AttnSmem<D>::alloc(a.gk.nT, a.topk, MODE == MODE_PAIR);
  if (cudaFuncSetAttribute(attn_fwd_kernel<D, MODE, F16, SAME, BNHD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           smem) !=
      cudaSuccess)
    return VSA_ERR_CUDA;
  const long long BH = 1ll * a.gq.B * a.gq.H;
  long long grid;
  if (MODE == MODE_SHARED) grid = BH * a.gq.nT * 2;                        // a t-half of a tile
  else if (MODE == MODE_TILE) grid = BH * a.gq.nT;                         // a tile
  else grid = BH * ((a.gq.nT + 1) / 2);                                    // a pair of tiles
  attn_fwd_kernel<D, MODE, F16, SAME, BNHD><<<static_cast<unsigned>(grid), kAttnThreads, smem, st>>>(mq, mk, mv, mo, a);
  return cudaGetLastError() == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

// Scratch of vsa_select_noalloc: file-scope device array, one per GPU that
// loads the library.  Host code must not pass `g_select_scratch` itself to a
// kernel (on the host it is only a stand-in symbol); its device address comes
// from cudaGetSymbolAddress, looked up once per device.
static __device__ __align__(256) float g_select_scratch[VSA_SELECT_NOALLOC_SCRATCH_BYTES / sizeof(float)];

static int select_scratch_ptr(float** out) {
  static SymbolCache cache;
  void* p = nullptr;
  const int rc = symbol_address(g_select_scratch, cache, &p);
  *out = static_cast<float*>(p);
  return rc;
}

// SAME: the key/value side has the query grid and tile (the kernel then
// reads one geometry; see kv_geom).
template <bool F16, bool SAME, bool BNHD>
static int dispatch_attn_d(int d, int mode, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                           const CUtensorMap& mo, const AttnArgs& a, cudaStream_t st) {
  if (d == 128) {
    if (mode == MODE_SHARED) return launch_attn<128, MODE_SHARED, F16, SAME, BNHD>(mq, mk, mv, mo, a, st);
    if (mode == MODE_TILE) return launch_attn<128, MODE_TILE, F16, SAME, BNHD>(mq, mk, mv, mo, a, st);
    return launch_attn<128, MODE_PAIR, F16, SAME, BNHD>(mq, mk, mv, mo, a, st);
  }
  if (mode == MODE_SHARED) return launch_attn<64, MODE_SHARED, F16, SAME, BNHD>(mq, mk, mv, mo, a, st);
  if (mode == MODE_TILE) return launch_attn<64, MODE_TILE, F16, SAME, BNHD>(mq, mk, mv, mo, a, st);
  return launch_attn<64, MODE_PAIR, F16, SAME, BNHD>(mq, mk, mv, mo, a, st);
}

template <bool F16>
static int dispatch_attn(int d, int mode, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                         const CUtensorMap& mo, const AttnArgs& a, cudaStream_t st) {
  const bool same = a.gq.T == a.gk.T && a.gq.Hh == a.gk.Hh && a.gq.W == a.gk.W && a.gq.tt == a.gk.tt &&
                    a.gq.th == a.gk.th && a.gq.tw == a.gk.tw;
  // the layout is a template parameter too: the producer's box coordinates
  // of the default layout then need no division (measured ~8% at 64-token tiles)
  if (a.gq.layout == VSA_LAYOUT_BNHD)
    return same ? dispatch_attn_d<F16, true, true>(d, mode, mq, mk, mv, mo, a, st)
                : dispatch_attn_d<F16, false, true>(d, mode, mq, mk, mv, mo, a, st);
  return same ? dispatch_attn_d<F16, true, false>(d, mode, mq, mk, mv, mo, a, st)
              : dispatch_attn_d<F16, false, false>(d, mode, mq, mk, mv, mo, a, st);
}

static int dispatch_select(const Geom& gq, const Geom& gk, const void* q, const void* k, int topk, int32_t* idx,
                           void* ws, cudaStream_t st, const void* v = nullptr, float scale_log2 = 0.f,
                           float* coarse = nullptr) {
  if (gq.d == 128) return gq.f16 ? launch_select<128, true>(gq, gk, q, k, v, topk, idx, ws, scale_log2, coarse, st)
                                 : launch_select<128, false>(gq, gk, q, k, v, topk, idx, ws, scale_log2, coarse, st);
  return gq.f16 ? launch_select<64, true>(gq, gk, q, k, v, topk, idx, ws, scale_log2, coarse, st)
                : launch_select<64, false>(gq, gk, q, k, v, topk, idx, ws, scale_log2, coarse, st);
}

static int tile_count_of(const Geom& g, int32_t* num_tiles, int32_t* tiles_per_axis) {
  *num_tiles = g.nT;
  if (tiles_per_axis != nullptr) {
    tiles_per_axis[0] = g.nTt;
    tiles_per_axis[1] = g.nTy;
    tiles_per_axis[2] = g.nTx;
  }
  return VSA_OK;
}

}  // namespace vsa

using namespace vsa;

extern "C" {

int vsa_tile_count(const vsa_shape* shape, int32_t* num_tiles, int32_t* tiles_per_axis) {
  if (num_tiles == nullptr) return VSA_ERR_INVALID_ARG;
  Geom gq, gk;
  const int rc = make_geoms(shape, &gq, &gk);
  return rc != VSA_OK ? rc : tile_count_of(gq, num_tiles, tiles_per_axis);
}

int vsa_kv_tile_count(const vsa_shape* shape, int32_t* num_tiles, int32_t* tiles_per_axis) {
  if (num_tiles == nullptr) return VSA_ERR_INVALID_ARG;
  Geom gq, gk;
  const int rc = make_geoms(shape, &gq, &gk);
  return rc != VSA_OK ? rc : tile_count_of(gk, num_tiles, tiles_per_axis);
}

int vsa_topk_from_sparsity(const vsa_shape* shape, float sparsity, int32_t* topk) {
  if (topk == nullptr) return VSA_ERR_INVALID_ARG;
  Geom gq, gk;
  const int rc = make_geoms(shape, &gq, &gk);
  if (rc != VSA_OK) return rc;
  if (!(sparsity >= 0.f && sparsity < 1.f)) return VSA_ERR_TOPK_RANGE;
  const double keep = (1.0 - static_cast<double>(sparsity)) * gk.nT;
  long long k = static_cast<long long>(std::floor(keep + 0.5));
  if (k < 1) k = 1;
  if (k < gk.prefix) k = gk.prefix;
  if (k > gk.nT) k = gk.nT;
  *topk = static_cast<int32_t>(k);
  return VSA_OK;
}

size_t vsa_select_workspace_bytes(const vsa_shape* shape) {
  Geom gq, gk;
  if (make_geoms(shape, &gq, &gk) != VSA_OK) return 0;
  return select_workspace_bytes(gq, gk);
}

int vsa_select(const vsa_shape* shape, const void* q, const void* k, int32_t topk, int32_t* idx_out,
               void* workspace, size_t workspace_bytes, void* stream) {
  Geom gq, gk;
  int rc = make_geoms(shape, &gq, &gk);
  if (rc != VSA_OK) return rc;
  if (q == nullptr || k == nullptr || idx_out == nullptr) return VSA_ERR_INVALID_ARG;
  if (topk <= 0 || topk > gk.nT || topk < gk.prefix) return VSA_ERR_TOPK_RANGE;
  if (!aligned16(q) || !aligned16(k) || !aligned16(workspace) || (reinterpret_cast<uintptr_t>(idx_out) & 3u))
    return VSA_ERR_ALIGNMENT;
  if (workspace == nullptr || workspace_bytes < select_workspace_bytes(gq, gk)) return VSA_ERR_WORKSPACE;
  if ((rc = check_arch()) != VSA_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return dispatch_select(gq, gk, q, k, topk, idx_out, workspace, st);
}

int vsa_select_noalloc(const vsa_shape* shape, const void* q, const void* k, int32_t topk, int32_t* idx_out,
                       void* stream) {
  Geom gq, gk;
  int rc = make_geoms(shape, &gq, &gk);
  if (rc != VSA_OK) return rc;
  if (q == nullptr || k == nullptr || idx_out == nullptr) return VSA_ERR_INVALID_ARG;
  if (topk <= 0 || topk > gk.nT || topk < gk.prefix) return VSA_ERR_TOPK_RANGE;
  if (!aligned16(q) || !aligned16(k) || (reinterpret_cast<uintptr_t>(idx_out) & 3u)) return VSA_ERR_ALIGNMENT;
  if (select_workspace_bytes(gq, gk) > VSA_SELECT_NOALLOC_SCRATCH_BYTES) return VSA_ERR_WORKSPACE;
  if ((rc = check_arch()) != VSA_OK) return rc;
  float* ws = nullptr;
  if ((rc = select_scratch_ptr(&ws)) != VSA_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return dispatch_select(gq, gk, q, k, topk, idx_out, ws, st);
}

}  // extern "C"

namespace vsa {

// vsa_attn_fwd and its gated form (gate, coarse: both or neither).
static int attn_fwd_impl(const vsa_shape* shape, const void* q, const void* k, const void* v, const int32_t* idx,
                         int32_t topk, float softmax_scale, const float* coarse, const void* gate, void* o,
                         float* lse, void* stream) {
  Geom gq, gk;
  int rc = make_geoms(shape, &gq, &gk);
  if (rc != VSA_OK) return rc;
  if (q == nullptr || k == nullptr || v == nullptr || idx == nullptr || o == nullptr || lse == nullptr)
    return VSA_ERR_INVALID_ARG;
  if ((gate == nullptr) != (coarse == nullptr)) return VSA_ERR_INVALID_ARG;
  if (!(softmax_scale > 0.f) || !std::isfinite(softmax_scale)) return VSA_ERR_INVALID_ARG;
  if (topk <= 0 || topk > gk.nT) return VSA_ERR_TOPK_RANGE;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      (reinterpret_cast<uintptr_t>(idx) & 3u) || (reinterpret_cast<uintptr_t>(lse) & 3u) ||
      (gate != nullptr && (!aligned16(gate) || !aligned16(coarse))))
    return VSA_ERR_ALIGNMENT;
  const int vol = gq.vol;                    // equal on both sides
  const int mode = vol == 256 ? MODE_SHARED : (vol == 128 ? MODE_TILE : MODE_PAIR);
  const int smem = gq.d == 128 ? AttnSmem<128>::alloc(gk.nT, topk, mode == MODE_PAIR)
                               : AttnSmem<64>::alloc(gk.nT, topk, mode == MODE_PAIR);
  if (smem > kMaxSmemPerBlock) return VSA_ERR_TOO_LARGE;
  if ((rc = check_arch()) != VSA_OK) return rc;

  const bool shared = (vol == 256);
  AttnArgs a;
  a.gq = gq;
  a.gk = gk;
  a.topk = topk;
  a.scale_log2 = softmax_scale * 1.4426950408889634f;
  a.idx = idx;
  a.o = static_cast<uint16_t*>(o);
  a.lse = lse;
  a.err = device_error_ptr();
  a.box_tq = shared ? gq.tt / 2 : gq.tt;
  a.box_tk = shared ? gk.tt / 2 : gk.tt;
  a.gate = static_cast<const uint16_t*>(gate);
  a.coarse = coarse;
  if (a.err == nullptr) return VSA_ERR_CUDA;
  CUtensorMap mq, mk, mv, mo;
  const bool f16 = gq.f16 != 0;
  if ((rc = encode_qkv_map(&mq, q, gq, a.box_tq, f16)) != VSA_OK ||
      (rc = encode_qkv_map(&mk, k, gk, a.box_tk, f16)) != VSA_OK ||
      (rc = encode_qkv_map(&mv, v, gk, a.box_tk, f16)) != VSA_OK ||
      (rc = encode_o_map(&mo, o, gq, a.box_tq, f16)) != VSA_OK)
    return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return f16 ? dispatch_attn<true>(gq.d, mode, mq, mk, mv, mo, a, st)
             : dispatch_attn<false>(gq.d, mode, mq, mk, mv, mo, a, st);
}

// ----------------------------------------------------- host-to-host forward
// Chunks of `c` heads: [B, H, N, d] holds a head's tokens contiguously and
// consecutive heads back to back, so a chunk is one contiguous range of
// (b, h) pairs; in [B, N, H, d] a chunk is c heads of one batch, a strided
// block copied with a 2-D copy into a dense [N, c, d] buffer.  Two buffer
// sets in the caller's workspace; uploads, kernels and downloads run on
// three streams of the library so chunk i+1's upload and chunk i-1's
// download overlap chunk i's kernels.
static size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct HostPlan {
  int c;                     // heads per chunk
  size_t q, k, o, lse, idx, sel, set;   // bytes of each buffer of one set (256-aligned), and of the set
};

static HostPlan host_plan(const vsa_shape* s, const Geom& gq, const Geom& gk, int topk, int chunk_heads) {
  HostPlan p;
  const int maxc = s->layout == VSA_LAYOUT_BNHD ? s->H : s->B * s->H;
  p.c = chunk_heads < 1 ? 1 : (chunk_heads > maxc ? maxc : chunk_heads);
  const size_t Nq = static_cast<size_t>(gq.T) * gq.Hh * gq.W, Nk = static_cast<size_t>(gk.T) * gk.Hh * gk.W;
  const size_t c = static_cast<size_t>(p.c), d = static_cast<size_t>(s->d);
  Geom cq = gq, ck = gk;
  cq.B = ck.B = 1;
  cq.H = ck.H = p.c;
  p.q = align256(c * Nq * d * 2);
  p.k = align256(c * Nk * d * 2);
  p.o = p.q;
  p.lse = align256(c * Nq * 4);
  p.idx = align256(c * static_cast<size_t>(gq.nT) * topk * 4);
  p.sel = align256(select_workspace_bytes(cq, ck));
  p.set = p.q + 2 * p.k + p.o + p.lse + p.idx + p.sel;
  return p;
}

struct HostStreams {
  cudaStream_t in, comp, out;
  cudaEvent_t start, ev_in[2], ev_comp[2], ev_out[2], done_in, done_comp, done_out;
  std::atomic<bool> ready{false};
};

// The three streams and their events, created once per device (the first
// host-to-host call on a device creates them: driver objects, no device
// memory of the caller's).
static int host_streams(HostStreams** out, std::mutex** mu) {
  static HostStreams hs[kMaxDevices];
  static std::mutex mus[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return VSA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return VSA_ERR_ARCH;
  *mu = &mus[dev];
  HostStreams& h = hs[dev];
  if (!h.ready) {
    std::lock_guard<std::mutex> lock(mus[dev]);
    if (!h.ready) {
      bool ok = cudaStreamCreateWithFlags(&h.in, cudaStreamNonBlocking) == cudaSuccess &&
                cudaStreamCreateWithFlags(&h.comp, cudaStreamNonBlocking) == cudaSuccess &&
                cudaStreamCreateWithFlags(&h.out, cudaStreamNonBlocking) == cudaSuccess;
      cudaEvent_t* evs[] = {&h.start, &h.ev_in[0], &h.ev_in[1], &h.ev_comp[0], &h.ev_comp[1], &h.ev_out[0],
                            &h.ev_out[1], &h.done_in, &h.done_comp, &h.done_out};
      for (cudaEvent_t* e : evs) ok = ok && cudaEventCreateWithFlags(e, cudaEventDisableTiming) == cudaSuccess;
      if (!ok) return VSA_ERR_CUDA;
      h.ready = true;
    }
  }
  *out = &h;
  return VSA_OK;
}

}  // namespace vsa

extern "C" {

int vsa_attn_fwd(const vsa_shape* shape, const void* q, const void* k, const void* v, const int32_t* idx,
                 int32_t topk, float softmax_scale, void* o, float* lse, void* stream) {
  return attn_fwd_impl(shape, q, k, v, idx, topk, softmax_scale, nullptr, nullptr, o, lse, stream);
}

size_t vsa_select_coarse_workspace_bytes(const vsa_shape* shape) {
  Geom gq, gk;
  if (make_geoms(shape, &gq, &gk) != VSA_OK) return 0;
  return coarse_workspace_bytes(gq, gk);
}

int vsa_select_coarse(const vsa_shape* shape, const void* q, const void* k, const void* v, int32_t topk,
                      float softmax_scale, int32_t* idx_out, float* coarse_out, void* workspace,
                      size_t workspace_bytes, void* stream) {
  Geom gq, gk;
  int rc = make_geoms(shape, &gq, &gk);
  if (rc != VSA_OK) return rc;
  if (q == nullptr || k == nullptr || v == nullptr || idx_out == nullptr || coarse_out == nullptr)
    return VSA_ERR_INVALID_ARG;
  if (!(softmax_scale > 0.f) || !std::isfinite(softmax_scale)) return VSA_ERR_INVALID_ARG;
  if (topk <= 0 || topk > gk.nT || topk < gk.prefix) return VSA_ERR_TOPK_RANGE;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(workspace) ||
      (reinterpret_cast<uintptr_t>(idx_out) & 3u) || (reinterpret_cast<uintptr_t>(coarse_out) & 3u))
    return VSA_ERR_ALIGNMENT;
  if (workspace == nullptr || workspace_bytes < coarse_workspace_bytes(gq, gk)) return VSA_ERR_WORKSPACE;
  if ((rc = check_arch()) != VSA_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return dispatch_select(gq, gk, q, k, topk, idx_out, workspace, st, v, softmax_scale * 1.4426950408889634f,
                         coarse_out);
}

int vsa_attn_fwd_gated(const vsa_shape* shape, const void* q, const void* k, const void* v, const int32_t* idx,
                       int32_t topk, float softmax_scale, const float* coarse, const void* gate, void* o,
                       float* lse, void* stream) {
  if (coarse == nullptr || gate == nullptr) return VSA_ERR_INVALID_ARG;
  return attn_fwd_impl(shape, q, k, v, idx, topk, softmax_scale, coarse, gate, o, lse, stream);
}

size_t vsa_forward_host_workspace_bytes(const vsa_shape* shape, int32_t topk, int32_t chunk_heads) {
  Geom gq, gk;
  if (make_geoms(shape, &gq, &gk) != VSA_OK || topk <= 0 || topk > gk.nT) return 0;
  return 2 * host_plan(shape, gq, gk, topk, chunk_heads).set;
}

int vsa_forward_host(const vsa_shape* shape, const void* q, const void* k, const void* v, int32_t topk,
                     float softmax_scale, void* o, float* lse, int32_t* idx, int32_t chunk_heads, void* workspace,
                     size_t workspace_bytes, void* stream) {
  Geom gq, gk;
  int rc = make_geoms(shape, &gq, &gk);
  if (rc != VSA_OK) return rc;
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr || lse == nullptr || idx == nullptr)
    return VSA_ERR_INVALID_ARG;
  if (!(softmax_scale > 0.f) || !std::isfinite(softmax_scale)) return VSA_ERR_INVALID_ARG;
  if (topk <= 0 || topk > gk.nT || topk < gk.prefix) return VSA_ERR_TOPK_RANGE;
  if (!aligned16(workspace)) return VSA_ERR_ALIGNMENT;
  const HostPlan pl = host_plan(shape, gq, gk, topk, chunk_heads);
  if (workspace == nullptr || workspace_bytes < 2 * pl.set) return VSA_ERR_WORKSPACE;
  if ((rc = check_arch()) != VSA_OK) return rc;
  HostStreams* hs = nullptr;
  std::mutex* mu = nullptr;
  if ((rc = host_streams(&hs, &mu)) != VSA_OK) return rc;
  std::lock_guard<std::mutex> lock(*mu);
  cudaStream_t caller = static_cast<cudaStream_t>(stream);
  const bool bnhd = shape->layout == VSA_LAYOUT_BNHD;
  const size_t Nq = static_cast<size_t>(gq.T) * gq.Hh * gq.W, Nk = static_cast<size_t>(gk.T) * gk.Hh * gk.W;
  const size_t d = static_cast<size_t>(shape->d), es = 2;
  const int B = shape->B, H = shape->H;
  // chunk list: (first (b, h) pair as b * H + h, heads); in [B, N, H, d] chunks stay within a batch
  const int per_b = bnhd ? (H + pl.c - 1) / pl.c : 0;
  const int nchunk = bnhd ? B * per_b : (B * H + pl.c - 1) / pl.c;
  auto ck = [&](int i, int* bh0, int* nh) {
    if (bnhd) {
      const int b = i / per_b, h0 = (i % per_b) * pl.c;
      *bh0 = b * H + h0;
      *nh = (H - h0 < pl.c) ? H - h0 : pl.c;
    } else {
      *bh0 = i * pl.c;
      *nh = (B * H - *bh0 < pl.c) ? B * H - *bh0 : pl.c;
    }
  };
  auto fail = [&]() { return VSA_ERR_CUDA; };
  if (cudaEventRecord(hs->start, caller) != cudaSuccess || cudaStreamWaitEvent(hs->in, hs->start, 0) != cudaSuccess ||
      cudaStreamWaitEvent(hs->comp, hs->start, 0) != cudaSuccess ||
      cudaStreamWaitEvent(hs->out, hs->start, 0) != cudaSuccess)
    return fail();
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  const unsigned char* hq = static_cast<const unsigned char*>(q);
  const unsigned char* hk = static_cast<const unsigned char*>(k);
  const unsigned char* hv = static_cast<const unsigned char*>(v);
  unsigned char* ho = static_cast<unsigned char*>(o);
  for (int i = 0; i < nchunk; ++i) {
    const int bs = i & 1;
    int bh0, nh;
    ck(i, &bh0, &nh);
    unsigned char* set = ws + bs * pl.set;
    unsigned char *dq = set, *dk = dq + pl.q, *dv = dk + pl.k, *dob = dv + pl.k;
    float* dl = reinterpret_cast<float*>(dob + pl.o);
    int32_t* di = reinterpret_cast<int32_t*>(dob + pl.o + pl.lse);
    void* dsel = dob + pl.o + pl.lse + pl.idx;
    const size_t nhs = static_cast<size_t>(nh);
    // uploads (after this buffer set's previous downloads)
    if (i >= 2 && cudaStreamWaitEvent(hs->in, hs->ev_out[bs], 0) != cudaSuccess) return fail();
    if (!bnhd) {
      const size_t oq = static_cast<size_t>(bh0) * Nq * d * es, okv = static_cast<size_t>(bh0) * Nk * d * es;
      if (cudaMemcpyAsync(dq, hq + oq, nhs * Nq * d * es, cudaMemcpyHostToDevice, hs->in) != cudaSuccess ||
          cudaMemcpyAsync(dk, hk + okv, nhs * Nk * d * es, cudaMemcpyHostToDevice, hs->in) != cudaSuccess ||
          cudaMemcpyAsync(dv, hv + okv, nhs * Nk * d * es, cudaMemcpyHostToDevice, hs->in) != cudaSuccess)
        return fail();
    } else {
      const int b = bh0 / H, h0 = bh0 % H;
      const size_t row = static_cast<size_t>(H) * d * es, w = nhs * d * es;
      const size_t oq = (static_cast<size_t>(b) * Nq * H + h0) * d * es;
      const size_t okv = (static_cast<size_t>(b) * Nk * H + h0) * d * es;
      if (cudaMemcpy2DAsync(dq, w, hq + oq, row, w, Nq, cudaMemcpyHostToDevice, hs->in) != cudaSuccess ||
          cudaMemcpy2DAsync(dk, w, hk + okv, row, w, Nk, cudaMemcpyHostToDevice, hs->in) != cudaSuccess ||
          cudaMemcpy2DAsync(dv, w, hv + okv, row, w, Nk, cudaMemcpyHostToDevice, hs->in) != cudaSuccess)
        return fail();
    }
    if (cudaEventRecord(hs->ev_in[bs], hs->in) != cudaSuccess) return fail();
    // kernels on the chunk: the same shape with B = 1 and H = nh
    vsa_shape cs = *shape;
    cs.B = 1;
    cs.H = nh;
    Geom cq, ckv;
    if ((rc = make_geoms(&cs, &cq, &ckv)) != VSA_OK) return rc;
    if (cudaStreamWaitEvent(hs->comp, hs->ev_in[bs], 0) != cudaSuccess) return fail();
    if ((rc = dispatch_select(cq, ckv, dq, dk, topk, di, dsel, hs->comp)) != VSA_OK) return rc;
    if ((rc = attn_fwd_impl(&cs, dq, dk, dv, di, topk, softmax_scale, nullptr, nullptr, dob, dl, hs->comp)) !=
        VSA_OK)
      return rc;
    if (cudaEventRecord(hs->ev_comp[bs], hs->comp) != cudaSuccess) return fail();
    // downloads
    if (cudaStreamWaitEvent(hs->out, hs->ev_comp[bs], 0) != cudaSuccess) return fail();
    const size_t ol = static_cast<size_t>(bh0) * Nq * 4;
    const size_t oi = static_cast<size_t>(bh0) * gq.nT * topk * 4;
    if (!bnhd) {
      if (cudaMemcpyAsync(ho + static_cast<size_t>(bh0) * Nq * d * es, dob, nhs * Nq * d * es, cudaMemcpyDeviceToHost,
                          hs->out) != cudaSuccess)
        return fail();
    } else {
      const int b = bh0 / H, h0 = bh0 % H;
      const size_t row = static_cast<size_t>(H) * d * es, w = nhs * d * es;
      if (cudaMemcpy2DAsync(ho + (static_cast<size_t>(b) * Nq * H + h0) * d * es, row, dob, w, w, Nq,
                            cudaMemcpyDeviceToHost, hs->out) != cudaSuccess)
        return fail();
    }
    if (cudaMemcpyAsync(reinterpret_cast<unsigned char*>(lse) + ol, dl, nhs * Nq * 4, cudaMemcpyDeviceToHost,
                        hs->out) != cudaSuccess ||
        cudaMemcpyAsync(reinterpret_cast<unsigned char*>(idx) + oi, di, nhs * gq.nT * topk * 4,
                        cudaMemcpyDeviceToHost, hs->out) != cudaSuccess ||
        cudaEventRecord(hs->ev_out[bs], hs->out) != cudaSuccess)
      return fail();
  }
  // the caller's stream waits for all of it
  if (cudaEventRecord(hs->done_in, hs->in) != cudaSuccess || cudaEventRecord(hs->done_comp, hs->comp) != cudaSuccess ||
      cudaEventRecord(hs->done_out, hs->out) != cudaSuccess || cudaStreamWaitEvent(caller, hs->done_in, 0) != cudaSuccess ||
      cudaStreamWaitEvent(caller, hs->done_comp, 0) != cudaSuccess ||
      cudaStreamWaitEvent(caller, hs->done_out, 0) != cudaSuccess)
    return fail();
  return VSA_OK;
}

int vsa_device_error(uint32_t* code, int32_t reset) {
  if (code == nullptr) return VSA_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return VSA_ERR_CUDA;
  unsigned int h = 0;
  if (cudaMemcpyFromSymbol(&h, g_device_error, sizeof(h)) != cudaSuccess) return VSA_ERR_CUDA;
  *code = h;
  if (reset) {
    const unsigned int z = 0;
    if (cudaMemcpyToSymbol(g_device_error, &z, sizeof(z)) != cudaSuccess) return VSA_ERR_CUDA;
  }
  return VSA_OK;
}

const char* vsa_status_string(int32_t status) {
  switch (status) {
    case VSA_OK: return "VSA_OK";
    case VSA_ERR_INVALID_ARG: return "VSA_ERR_INVALID_ARG";
    case VSA_ERR_TOPK_RANGE: return "VSA_ERR_TOPK_RANGE";
    case VSA_ERR_UNSUPPORTED: return "VSA_ERR_UNSUPPORTED";
    case VSA_ERR_ALIGNMENT: return "VSA_ERR_ALIGNMENT";
    case VSA_ERR_WORKSPACE: return "VSA_ERR_WORKSPACE";
    case VSA_ERR_ARCH: return "VSA_ERR_ARCH";
    case VSA_ERR_CUDA: return "VSA_ERR_CUDA";
    case VSA_ERR_TOO_LARGE: return "VSA_ERR_TOO_LARGE";
    default: return "VSA_ERR_UNKNOWN";
  }
}

}  // extern "C"
