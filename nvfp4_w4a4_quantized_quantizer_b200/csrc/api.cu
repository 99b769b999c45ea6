// api.cu -- the C ABI declared in include/nvfp4.h.
//
// Host side of the NVFP4 W4A4 linear layer: argument validation (before any
// CUDA call), per-device capability checks, TMA descriptor encoding (cached
// per pointer and shape), kernel selection and launch.  The library never
// allocates or frees device memory; every buffer belongs to the caller.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <unordered_map>

#include "nvfp4.h"
#include "gdn.cuh"
#include "gemm.cuh"
#include "quantize.cuh"

namespace {

using nvfp4::SegTable;

// --------------------------------------------------------------- settings
uint64_t read_env_wait_ns() {
  const char* e = std::getenv("NVFP4_SPIN_LIMIT_NS");
  if (e != nullptr) {
    const unsigned long long v = std::strtoull(e, nullptr, 10);
    if (v > 0) return v;
  }
  return 2000000000ull;
}

uint64_t g_wait_ns = read_env_wait_ns();
int g_gemm_path = 0;
bool g_overlap = false;

// Launch with programmatic stream serialization when launch overlap is on:
// the kernel may then start before the kernel ahead of it on the stream has
// finished (it waits for it with griddepcontrol.wait where it must).
template <typename Kernel, typename... Args>
nvfp4_status launch_maybe_overlapped(Kernel kernel, dim3 grid, dim3 block, int smem,
                                     cudaStream_t st, Args... args) {
  if (!g_overlap) {
    kernel<<<grid, block, smem, st>>>(args...);
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
  }
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kernel, args...) != cudaSuccess) {
    cudaGetLastError();
    return NVFP4_ERR_CUDA;
  }
  return NVFP4_OK;
}

// ----------------------------------------------------------- device info
constexpr int MAX_DEVICES = 64;
struct DeviceInfo {
  bool probed = false;
  bool supported = false;
  int sms = 0;
  bool attr_tc = false;
  bool attr_tc2 = false;
  bool attr_tc2_swiglu = false;
  bool attr_gdn = false;
  int quant_blocks = 0;   // resident k_quantize blocks per SM
  int pairs = 0;          // co-resident clusters of two CTAs of k_gemm_tc<2>
  int swiglu_pairs = 0;   // the same for k_gemm_tc<2, true>
  bool attr_small[3] = {false, false, false};
};
DeviceInfo g_dev[MAX_DEVICES];
std::mutex g_mu;

nvfp4_status current_device(int* dev_out, DeviceInfo** info_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return NVFP4_ERR_CUDA;
  }
  if (dev < 0 || dev >= MAX_DEVICES) return NVFP4_ERR_UNSUPPORTED_DEVICE;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.probed) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      return NVFP4_ERR_CUDA;
    }
    d.probed = true;
    d.supported = (major == 10 && minor == 0);
    d.sms = sms;
  }
  if (!d.supported) return NVFP4_ERR_UNSUPPORTED_DEVICE;
  *dev_out = dev;
  *info_out = &d;
  return NVFP4_OK;
}

nvfp4_status check_launch() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

// ------------------------------------------------------------ tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
    else
      cudaGetLastError();
  });
  return fn;
}

struct MapKey {
  const void* ptr;
  int64_t rows, row_bytes;
  int box_rows;
  int dev;
  bool operator==(const MapKey& o) const {
    return ptr == o.ptr && rows == o.rows && row_bytes == o.row_bytes && box_rows == o.box_rows &&
           dev == o.dev;
  }
};
struct MapKeyHash {
  size_t operator()(const MapKey& k) const {
    size_t h = std::hash<const void*>()(k.ptr);
    h ^= std::hash<int64_t>()(k.rows * 1315423911ll + k.row_bytes) + 0x9e3779b97f4a7c15ull +
         (h << 6) + (h >> 2);
    h ^= static_cast<size_t>(k.box_rows * 131 + k.dev);
    return h;
  }
};
std::unordered_map<MapKey, CUtensorMap, MapKeyHash> g_maps;
std::mutex g_map_mu;

// 2-D uint8 map over a [rows, row_bytes] code matrix, box = 128 bytes x
// box_rows rows, 128-byte swizzle, out-of-range elements read as zero.
nvfp4_status code_map(const void* ptr, int64_t rows, int64_t row_bytes, int box_rows, int dev,
                      CUtensorMap* out) {
  const MapKey key{ptr, rows, row_bytes, box_rows, dev};
  {
    std::lock_guard<std::mutex> lk(g_map_mu);
    auto it = g_maps.find(key);
    if (it != g_maps.end()) {
      *out = it->second;
      return NVFP4_OK;
    }
  }
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return NVFP4_ERR_CUDA;
  CUtensorMap m;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(row_bytes), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(row_bytes)};
  const cuuint32_t box[2] = {128u, static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1u, 1u};
  const CUresult r = fn(&m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return NVFP4_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_map_mu);
  if (g_maps.size() > 4096) g_maps.clear();
  g_maps[key] = m;
  *out = m;
  return NVFP4_OK;
}

// 3-D uint64 map over a scale buffer in the 128x4 atom layout, viewed as
// [row blocks of 128][K/64 atoms][64 x 8 bytes]; box = the 4 atoms of one
// 256-element k-tile for `box_blocks` row blocks.  Atoms past K or past the
// last row block read as zero.
nvfp4_status scale_map(const void* ptr, int64_t rows, int64_t K, int box_blocks, int dev,
                       CUtensorMap* out) {
  const MapKey key{ptr, rows, K, -box_blocks, dev};
  {
    std::lock_guard<std::mutex> lk(g_map_mu);
    auto it = g_maps.find(key);
    if (it != g_maps.end()) {
      *out = it->second;
      return NVFP4_OK;
    }
  }
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return NVFP4_ERR_CUDA;
  CUtensorMap m;
  const int64_t kb4 = K / 64;
  const int64_t blocks = (rows + 127) / 128;
  const cuuint64_t dims[3] = {64u, static_cast<cuuint64_t>(kb4), static_cast<cuuint64_t>(blocks)};
  const cuuint64_t strides[2] = {512u, static_cast<cuuint64_t>(kb4 * 512)};
  const cuuint32_t box[3] = {64u, 4u, static_cast<cuuint32_t>(box_blocks)};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  const CUresult r = fn(&m, CU_TENSOR_MAP_DATA_TYPE_UINT64, 3, const_cast<void*>(ptr), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return NVFP4_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_map_mu);
  if (g_maps.size() > 4096) g_maps.clear();
  g_maps[key] = m;
  *out = m;
  return NVFP4_OK;
}

// ------------------------------------------------------------- validation
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr int64_t kMaxDim = (1ll << 31) - 1;

// One stream-K partial tile (a workspace slot): 2 CTAs x 128 rows x 256
// columns of fp32.
constexpr size_t kPartialBytes = 2ull * nvfp4::tc::BM * nvfp4::tc::BN * 4;

nvfp4_status check_bf16_matrix(const void* x, int64_t R, int64_t K, int64_t ld) {
  if (x == nullptr) return NVFP4_ERR_INVALID_ARG;
  if (R < 0 || K < 64 || K % 64 != 0 || R > kMaxDim || K > kMaxDim) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (ld < K) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(x) || ld % 8 != 0) return NVFP4_ERR_ALIGNMENT;
  return NVFP4_OK;
}

bool good_scale(float s) { return std::isfinite(s) && s > 0.0f; }

int64_t pad128(int64_t r) { return (r + 127) / 128 * 128; }

int grid_for(int64_t work_items, int64_t per_block, int cap) {
  int64_t b = (work_items + per_block - 1) / per_block;
  if (b < 1) b = 1;
  if (b > cap) b = cap;
  return static_cast<int>(b);
}

nvfp4_status launch_quantize(const void* x, int64_t rows, int64_t K, int64_t ld, int64_t row0,
                             float gs, void* codes, void* scales, int64_t pad_from,
                             int64_t pad_to, DeviceInfo* info, cudaStream_t st) {
  nvfp4::QuantArgs a;
  a.x = static_cast<const __nv_bfloat16*>(x);
  a.rows = rows;
  a.K = K;
  a.ldx = ld;
  a.row0 = row0;
  a.gs = gs;
  a.codes = static_cast<uint8_t*>(codes);
  a.scales = static_cast<uint8_t*>(scales);
  a.pad_from = pad_from;
  a.pad_to = pad_to;
  // r[s] = fp32(1 / fp32(s_dec * gs)): IEEE fp32 host arithmetic rounds like
  // the device's correctly rounded reciprocal; s_dec is exact in fp32
  for (int code = 0; code < 128; ++code) {
    const int e = (code >> 3) & 0xF, m = code & 7;
    const float sdec = (e == 0) ? static_cast<float>(m) * 0.001953125f
                                : std::ldexp(1.0f + static_cast<float>(m) / 8.0f, e - 7);
    volatile float p = sdec * gs;   // volatile: keep the two fp32 roundings separate
    a.rtab[code] = (sdec == 0.0f || code == 127) ? 0.0f : 1.0f / p;
  }
  a.wait_ns = g_wait_ns;
  const int64_t units = rows * ((K + nvfp4::QUANT_UNIT - 1) / nvfp4::QUANT_UNIT);
  if (units == 0 && pad_to <= pad_from) return NVFP4_OK;
  constexpr int smem = nvfp4::QUANT_SMEM + nvfp4::QUANT_BAR_BYTES;
  if (info->quant_blocks == 0) {
    int blocks = 0;
    if (cudaFuncSetAttribute(nvfp4::k_quantize, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks, nvfp4::k_quantize,
                                                      nvfp4::QUANT_THREADS, smem) != cudaSuccess ||
        blocks < 1) {
      cudaGetLastError();
      return NVFP4_ERR_CUDA;
    }
    info->quant_blocks = blocks;
  }
  // persistent: one wave of resident blocks, each warp striding over the units
  const int grid = grid_for(units, nvfp4::QUANT_WARPS, info->sms * info->quant_blocks);
  return launch_maybe_overlapped(nvfp4::k_quantize, dim3(grid), dim3(nvfp4::QUANT_THREADS), smem,
                                 st, a);
}

nvfp4_status launch_amax(const void* x, int64_t rows, int64_t K, int64_t ld, float* out, int sms,
                         cudaStream_t st) {
  if (cudaMemsetAsync(out, 0, sizeof(float), st) != cudaSuccess) return NVFP4_ERR_CUDA;
  if (rows == 0) return NVFP4_OK;
  const int grid = grid_for(rows, nvfp4::AMAX_THREADS / 32, sms * 4);
  nvfp4::k_amax<<<grid, nvfp4::AMAX_THREADS, 0, st>>>(static_cast<const __nv_bfloat16*>(x), rows,
                                                       K, ld, out);
  return check_launch();
}

nvfp4_status build_segments(const nvfp4_segment* segs, int32_t nseg, int64_t N, SegTable* t) {
  if (segs == nullptr || nseg < 1 || nseg > NVFP4_MAX_SEGMENTS) return NVFP4_ERR_INVALID_ARG;
  std::memset(t, 0, sizeof(*t));
  t->nseg = nseg;
  for (int s = 0; s < nseg; ++s) {
    const nvfp4_segment& g = segs[s];
    if (s == 0 && g.n_offset != 0) return NVFP4_ERR_INVALID_ARG;
    if (s > 0 && g.n_offset <= segs[s - 1].n_offset) return NVFP4_ERR_INVALID_ARG;
    if (g.n_offset < 0 || g.n_offset >= N) return NVFP4_ERR_INVALID_ARG;
    if (g.n_offset % 16 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!good_scale(g.w_gs) || !good_scale(g.a_gs)) return NVFP4_ERR_INVALID_ARG;
    if (g.op < NVFP4_OP_NONE || g.op > NVFP4_OP_GDN_DECAY) return NVFP4_ERR_INVALID_ARG;
    if (g.op == NVFP4_OP_GDN_DECAY && (g.a_log == nullptr || g.dt_bias == nullptr))
      return NVFP4_ERR_INVALID_ARG;
    t->n_off[s] = static_cast<int>(g.n_offset);
    t->alpha[s] = g.a_gs * g.w_gs;  // fp32 product, round to nearest
    t->op[s] = g.op;
    t->a_log[s] = g.a_log;
    t->dt_bias[s] = g.dt_bias;
  }
  t->n_off[nseg] = static_cast<int>(N);
  return NVFP4_OK;
}

// ------------------------------------------ weight quantisation, no allocation
// Scratch of nvfp4_quantize_weight_noalloc: the per-module amax accumulators.
// A fixed array in the library's device image; every GPU that loads the
// library holds it (NVFP4_NOALLOC_MAX_SEGMENTS floats) until the process exits.
static __device__ __align__(256) float g_noalloc_amax[NVFP4_NOALLOC_MAX_SEGMENTS];

float* g_noalloc_ptr[MAX_DEVICES] = {};
std::mutex g_noalloc_mu;

// The array's device address on the current device.  In host code the name
// g_noalloc_amax is only a host-side stand-in, so the address is looked up
// once per device (with that device current) and cached.
nvfp4_status noalloc_scratch(float** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return NVFP4_ERR_CUDA;
  }
  if (dev < 0 || dev >= MAX_DEVICES) return NVFP4_ERR_UNSUPPORTED_DEVICE;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_amax);
    if (e != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return NVFP4_ERR_CUDA;
    }
    g_noalloc_ptr[dev] = static_cast<float*>(p);
  }
  *out = g_noalloc_ptr[dev];
  return NVFP4_OK;
}

// Launch configuration of a CTA-pair kernel (clusters of two CTAs, its
// dynamic shared memory, `st`, and with launch overlap on programmatic
// stream serialization); once per device and kernel, also the shared-memory
// attribute and the number of pairs that fit at once (clusters are placed
// within one GPC, so an SM count that is odd inside a GPC leaves an SM
// out).  attr (two entries) must outlive cfg.
template <typename Kernel>
nvfp4_status pair_config(Kernel kernel, DeviceInfo* info, bool* configured, int* max_pairs,
                         cudaStream_t st, cudaLaunchConfig_t* cfg, cudaLaunchAttribute* attr) {
  constexpr int smem = nvfp4::tc::Cfg<2>::SMEM_BYTES;
  *cfg = cudaLaunchConfig_t{};
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg->blockDim = dim3(nvfp4::tc::THREADS, 1, 1);
  cfg->dynamicSmemBytes = smem;
  cfg->stream = st;
  cfg->attrs = attr;
  cfg->numAttrs = 1;
  if (!*configured) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess) {
      cudaGetLastError();
      return NVFP4_ERR_CUDA;
    }
    cfg->gridDim = dim3(2 * (info->sms / 2), 1, 1);
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, kernel, cfg) != cudaSuccess || clusters < 1) {
      cudaGetLastError();
      return NVFP4_ERR_CUDA;
    }
    *max_pairs = clusters;
    *configured = true;
  }
  if (g_overlap) {
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg->numAttrs = 2;
  }
  return NVFP4_OK;
}

}  // namespace

// =================================================================== C ABI
extern "C" {

size_t nvfp4_codes_bytes(int64_t rows, int64_t K) {
  if (rows < 0 || K < 0) return 0;
  return static_cast<size_t>(rows) * static_cast<size_t>(K / 2);
}

size_t nvfp4_scale_bytes(int64_t rows, int64_t K) {
  if (rows < 0 || K < 0) return 0;
  return static_cast<size_t>(pad128(rows)) * static_cast<size_t>(K / 16);
}

float nvfp4_global_scale(float amax) { return amax > 0.0f ? amax / 2688.0f : 1.0f; }

const char* nvfp4_status_string(nvfp4_status s) {
  switch (s) {
    case NVFP4_OK: return "ok";
    case NVFP4_ERR_INVALID_ARG: return "invalid argument";
    case NVFP4_ERR_ALIGNMENT: return "pointer or leading dimension not 16-byte aligned";
    case NVFP4_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case NVFP4_ERR_CUDA: return "CUDA error";
    case NVFP4_ERR_TIMEOUT: return "bounded in-kernel wait timed out";
    case NVFP4_ERR_UNSUPPORTED_DEVICE: return "device is not compute capability 10.0 (sm_100a)";
  }
  return "unknown status";
}

nvfp4_status nvfp4_set_gemm_path(int32_t path) {
  if (path < 0 || path > 4) return NVFP4_ERR_INVALID_ARG;
  g_gemm_path = path;
  return NVFP4_OK;
}

nvfp4_status nvfp4_set_launch_overlap(int32_t on) {
  if (on != 0 && on != 1) return NVFP4_ERR_INVALID_ARG;
  g_overlap = (on == 1);
  return NVFP4_OK;
}

nvfp4_status nvfp4_set_wait_limit_ns(uint64_t limit_ns) {
  if (limit_ns == 0) return NVFP4_ERR_INVALID_ARG;
  g_wait_ns = limit_ns;
  return NVFP4_OK;
}

nvfp4_status nvfp4_last_device_error(nvfp4_stream_t stream, uint64_t* info) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return NVFP4_ERR_CUDA;
  }
  unsigned long long w = 0;
  if (cudaMemcpyFromSymbol(&w, nvfp4::g_error_word, sizeof(w)) != cudaSuccess) return NVFP4_ERR_CUDA;
  if (info != nullptr) *info = w;
  if (w == 0) return NVFP4_OK;
  const unsigned long long zero = 0;
  if (cudaMemcpyToSymbol(nvfp4::g_error_word, &zero, sizeof(zero)) != cudaSuccess)
    return NVFP4_ERR_CUDA;
  return NVFP4_ERR_TIMEOUT;
}

nvfp4_status nvfp4_amax(const void* x, int64_t R, int64_t K, int64_t ldx, float* amax_dev,
                        nvfp4_stream_t stream) {
  nvfp4_status st = check_bf16_matrix(x, R, K, ldx);
  if (st != NVFP4_OK) return st;
  if (amax_dev == nullptr) return NVFP4_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(amax_dev) & 3u) != 0) return NVFP4_ERR_ALIGNMENT;
  int dev;
  DeviceInfo* info;
  if ((st = current_device(&dev, &info)) != NVFP4_OK) return st;
  return launch_amax(x, R, K, ldx, amax_dev, info->sms, reinterpret_cast<cudaStream_t>(stream));
}

nvfp4_status nvfp4_quantize_act(const void* x, int64_t M, int64_t K, int64_t ldx, float a_gs,
                                void* codes, void* scales, nvfp4_stream_t stream) {
  nvfp4_status st = check_bf16_matrix(x, M, K, ldx);
  if (st != NVFP4_OK) return st;
  if (codes == nullptr || scales == nullptr) return NVFP4_ERR_INVALID_ARG;
  if (!aligned16(codes) || !aligned16(scales)) return NVFP4_ERR_ALIGNMENT;
  if (!good_scale(a_gs)) return NVFP4_ERR_INVALID_ARG;
  if (M == 0) return NVFP4_OK;
  int dev;
  DeviceInfo* info;
  if ((st = current_device(&dev, &info)) != NVFP4_OK) return st;
  return launch_quantize(x, M, K, ldx, 0, a_gs, codes, scales, M, pad128(M), info,
                         reinterpret_cast<cudaStream_t>(stream));
}

size_t nvfp4_quantize_weight_workspace_bytes(int32_t nseg) {
  if (nseg < 1) nseg = 1;
  return static_cast<size_t>((nseg * 4 + 255) / 256 * 256);
}

nvfp4_status nvfp4_quantize_weight(const void* w, int64_t N, int64_t K, int64_t ldw,
                                   const int64_t* seg_offsets, int32_t nseg, float* w_gs_out,
                                   void* codes, void* scales, void* workspace,
                                   nvfp4_stream_t stream) {
  nvfp4_status st = check_bf16_matrix(w, N, K, ldw);
  if (st != NVFP4_OK) return st;
  if (N < 16 || N % 16 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (codes == nullptr || scales == nullptr || w_gs_out == nullptr || workspace == nullptr)
    return NVFP4_ERR_INVALID_ARG;
  if (!aligned16(codes) || !aligned16(scales) || !aligned16(workspace)) return NVFP4_ERR_ALIGNMENT;
  if (nseg < 1 || nseg > NVFP4_MAX_SEGMENTS) return NVFP4_ERR_INVALID_ARG;
  if (seg_offsets == nullptr && nseg != 1) return NVFP4_ERR_INVALID_ARG;
  int64_t off[NVFP4_MAX_SEGMENTS + 1];
  for (int s = 0; s < nseg; ++s) {
    off[s] = seg_offsets ? seg_offsets[s] : 0;
    if (s == 0 && off[s] != 0) return NVFP4_ERR_INVALID_ARG;
    if (s > 0 && off[s] <= off[s - 1]) return NVFP4_ERR_INVALID_ARG;
    if (off[s] >= N) return NVFP4_ERR_INVALID_ARG;
    if (off[s] % 16 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  }
  off[nseg] = N;
  int dev;
  DeviceInfo* info;
  if ((st = current_device(&dev, &info)) != NVFP4_OK) return st;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  float* amax_dev = static_cast<float*>(workspace);
  const char* wb = static_cast<const char*>(w);
  for (int s = 0; s < nseg; ++s) {
    st = launch_amax(wb + off[s] * ldw * 2, off[s + 1] - off[s], K, ldw, amax_dev + s, info->sms, cs);
    if (st != NVFP4_OK) return st;
  }
  float amax[NVFP4_MAX_SEGMENTS];
  if (cudaMemcpyAsync(amax, amax_dev, nseg * sizeof(float), cudaMemcpyDeviceToHost, cs) !=
          cudaSuccess ||
      cudaStreamSynchronize(cs) != cudaSuccess) {
    cudaGetLastError();
    return NVFP4_ERR_CUDA;
  }
  for (int s = 0; s < nseg; ++s) {
    // an all-zero module quantises to zero codes under any scale; give it 1
    const float gs = nvfp4_global_scale(amax[s]);
    w_gs_out[s] = gs;
    const bool last = (s == nseg - 1);
    st = launch_quantize(wb + off[s] * ldw * 2, off[s + 1] - off[s], K, ldw, off[s], gs, codes,
                         scales, last ? N : 0, last ? pad128(N) : 0, info, cs);
    if (st != NVFP4_OK) return st;
  }
  // the codes and scales are complete on return, so that a GEMM launched
  // with launch overlap may stream them from its start
  if (cudaStreamSynchronize(cs) != cudaSuccess) {
    cudaGetLastError();
    return NVFP4_ERR_CUDA;
  }
  return NVFP4_OK;
}

nvfp4_status nvfp4_quantize_weight_noalloc(const void* w, int64_t N, int64_t K, int64_t ldw,
                                           const int64_t* seg_offsets, int32_t nseg,
                                           float* w_gs_out, void* codes, void* scales,
                                           nvfp4_stream_t stream) {
  if (nseg < 1 || nseg > NVFP4_NOALLOC_MAX_SEGMENTS) return NVFP4_ERR_INVALID_ARG;
  nvfp4_status st = check_bf16_matrix(w, N, K, ldw);
  if (st != NVFP4_OK) return st;
  if (codes == nullptr || scales == nullptr || w_gs_out == nullptr) return NVFP4_ERR_INVALID_ARG;
  int dev;
  DeviceInfo* info;
  if ((st = current_device(&dev, &info)) != NVFP4_OK) return st;
  float* scratch = nullptr;
  if ((st = noalloc_scratch(&scratch)) != NVFP4_OK) return st;
  // the workspace path clears each module's accumulator on `stream` before use
  return nvfp4_quantize_weight(w, N, K, ldw, seg_offsets, nseg, w_gs_out, codes, scales, scratch,
                               stream);
}

size_t nvfp4_gemm_workspace_bytes(void) {
  return static_cast<size_t>(NVFP4_GEMM_WS_COUNTER_BYTES) +
         static_cast<size_t>(NVFP4_GEMM_WS_MAX_UNITS) * kPartialBytes;
}

nvfp4_status nvfp4_fused_linear_ws(const void* a_codes, const void* a_scales, const void* w_codes,
                                   const void* w_scales, int64_t M, int64_t N, int64_t K,
                                   const nvfp4_segment* segs, int32_t nseg, void* y, int64_t ldy,
                                   nvfp4_out_dtype out_dtype, void* workspace,
                                   size_t workspace_bytes, nvfp4_stream_t stream) {
  if (a_codes == nullptr || a_scales == nullptr || w_codes == nullptr || w_scales == nullptr ||
      y == nullptr)
    return NVFP4_ERR_INVALID_ARG;
  if (workspace != nullptr && !aligned16(workspace)) return NVFP4_ERR_ALIGNMENT;
  if (out_dtype != NVFP4_OUT_BF16 && out_dtype != NVFP4_OUT_FP32) return NVFP4_ERR_INVALID_ARG;
  if (M < 0 || M > kMaxDim || N < 16 || N % 16 != 0 || N > kMaxDim || K < 64 || K % 64 != 0 ||
      K > kMaxDim || ldy < N)
    return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(a_codes) || !aligned16(a_scales) || !aligned16(w_codes) || !aligned16(w_scales) ||
      !aligned16(y))
    return NVFP4_ERR_ALIGNMENT;
  if (ldy % (out_dtype == NVFP4_OUT_FP32 ? 4 : 8) != 0) return NVFP4_ERR_ALIGNMENT;
  SegTable table;
  nvfp4_status st = build_segments(segs, nseg, N, &table);
  if (st != NVFP4_OK) return st;
  if (g_gemm_path == 2 && M > 64) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (M == 0) return NVFP4_OK;
  int dev;
  DeviceInfo* info;
  if ((st = current_device(&dev, &info)) != NVFP4_OK) return st;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);

  nvfp4::GemmArgs g;
  g.sfa = static_cast<const uint8_t*>(a_scales);
  g.sfb = static_cast<const uint8_t*>(w_scales);
  g.M = static_cast<int>(M);
  g.N = static_cast<int>(N);
  g.K = static_cast<int>(K);
  g.y = y;
  g.ldy = ldy;
  g.out_fp32 = (out_dtype == NVFP4_OUT_FP32);
  g.sector_stores = ((reinterpret_cast<uintptr_t>(y) & 31u) == 0) &&
                    ((ldy * (g.out_fp32 ? 4 : 2)) % 32 == 0);
  g.wait_ns = g_wait_ns;
  g.sk_tiles = 0;
  g.partial = nullptr;
  g.flags = nullptr;
  // Tile raster.  Consecutive CTAs (pairs) run tiles that share one operand
  // tile, and the rest of that operand is re-read from L2 for each of the
  // other operand's tiles.  By default they share weight tiles (M fastest),
  // which keeps the activations L2-resident; when the activation codes are
  // too large to stay in the 126 MB L2 (e.g. the MLP down projection's
  // 16384 x 17408 input, 143 MB) and the weights are smaller, they share
  // activation tiles instead, so the activations stream from HBM once.
  const int64_t a_bytes = M * (K / 2), w_bytes = N * (K / 2);
  g.n_fastest = (g_gemm_path == 4) || (a_bytes > (64ll << 20) && w_bytes < a_bytes);

  const bool small = (g_gemm_path == 2) || (g_gemm_path == 0 && M <= 64);
  if (small) {
    const int nt = M <= 16 ? 16 : (M <= 32 ? 32 : 64);
    const int which = nt == 16 ? 0 : (nt == 32 ? 1 : 2);
    CUtensorMap tw, tx;
    if ((st = code_map(w_codes, N, K / 2, nvfp4::sm::BW, dev, &tw)) != NVFP4_OK) return st;
    if ((st = code_map(a_codes, M, K / 2, nt, dev, &tx)) != NVFP4_OK) return st;
    const int grid = static_cast<int>((N + nvfp4::sm::BW - 1) / nvfp4::sm::BW);
    auto launch = [&](auto kernel, int smem) -> nvfp4_status {
      if (!info->attr_small[which]) {
        if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
            cudaSuccess)
          return NVFP4_ERR_CUDA;
        info->attr_small[which] = true;
      }
      return launch_maybe_overlapped(kernel, dim3(grid), dim3(nvfp4::sm::THREADS), smem, cs, tw,
                                     tx, g, table);
    };
    if (nt == 16) return launch(nvfp4::k_gemm_small<16>, nvfp4::sm::Cfg<16>::SMEM_BYTES);
    if (nt == 32) return launch(nvfp4::k_gemm_small<32>, nvfp4::sm::Cfg<32>::SMEM_BYTES);
    return launch(nvfp4::k_gemm_small<64>, nvfp4::sm::Cfg<64>::SMEM_BYTES);
  }

  const bool pair = (g_gemm_path >= 3) || (g_gemm_path == 0 && M > 128);
  CUtensorMap ta, tb, tsa, tsb;
  if ((st = code_map(a_codes, M, K / 2, nvfp4::tc::BM, dev, &ta)) != NVFP4_OK) return st;
  if ((st = code_map(w_codes, N, K / 2, nvfp4::tc::BN / (pair ? 2 : 1), dev, &tb)) != NVFP4_OK)
    return st;
  if ((st = scale_map(a_scales, M, K, 1, dev, &tsa)) != NVFP4_OK) return st;
  if ((st = scale_map(w_scales, N, K, 2, dev, &tsb)) != NVFP4_OK) return st;
  const int64_t num_n = (N + nvfp4::tc::BN - 1) / nvfp4::tc::BN;
  if (!pair) {
    constexpr int smem = nvfp4::tc::Cfg<1>::SMEM_BYTES;
    if (!info->attr_tc) {
      if (cudaFuncSetAttribute(nvfp4::k_gemm_tc<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               smem) != cudaSuccess)
        return NVFP4_ERR_CUDA;
      info->attr_tc = true;
    }
    const int64_t tiles = ((M + nvfp4::tc::BM - 1) / nvfp4::tc::BM) * num_n;
    const int grid = static_cast<int>(tiles < info->sms ? tiles : info->sms);
    return launch_maybe_overlapped(nvfp4::k_gemm_tc<1>, dim3(grid), dim3(nvfp4::tc::THREADS), smem,
                                   cs, ta, tb, tsa, tsb, g, table);
  }
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[2];
  if ((st = pair_config(nvfp4::k_gemm_tc<2>, info, &info->attr_tc2, &info->pairs, cs, &cfg,
                        attr)) != NVFP4_OK)
    return st;
  const int64_t tiles = ((M + 2 * nvfp4::tc::BM - 1) / (2 * nvfp4::tc::BM)) * num_n;
  const int pairs = static_cast<int>(tiles < info->pairs ? tiles : info->pairs);
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  // Stream-K tail: when the tiles are not a multiple of the pairs, the last
  // partial wave and one whole wave before it (sk_tiles = pairs + the
  // remainder) are cut into equal k-tile ranges, one per pair, instead of
  // leaving most pairs idle during the last wave.  Needs one workspace slot
  // per pair (the partial tile a pair publishes) and its flags.
  if (workspace != nullptr && tiles > pairs && tiles % pairs != 0) {
    const int64_t slots =
        workspace_bytes > NVFP4_GEMM_WS_COUNTER_BYTES
            ? static_cast<int64_t>((workspace_bytes - NVFP4_GEMM_WS_COUNTER_BYTES) / kPartialBytes)
            : 0;
    if (slots >= pairs && static_cast<int64_t>(pairs) * 2 * 4 <= NVFP4_GEMM_WS_COUNTER_BYTES) {
      g.sk_tiles = static_cast<int>(pairs + tiles % pairs);
      g.flags = static_cast<unsigned*>(workspace);
      g.partial = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                           NVFP4_GEMM_WS_COUNTER_BYTES);
    }
  }
  if (cudaLaunchKernelEx(&cfg, nvfp4::k_gemm_tc<2>, ta, tb, tsa, tsb, g, table) != cudaSuccess) {
    cudaGetLastError();
    return NVFP4_ERR_CUDA;
  }
  return check_launch();
}

int32_t nvfp4_noalloc_max_segments(void) { return NVFP4_NOALLOC_MAX_SEGMENTS; }

nvfp4_status nvfp4_fused_linear(const void* a_codes, const void* a_scales, const void* w_codes,
                                const void* w_scales, int64_t M, int64_t N, int64_t K,
                                const nvfp4_segment* segs, int32_t nseg, void* y, int64_t ldy,
                                nvfp4_out_dtype out_dtype, nvfp4_stream_t stream) {
  return nvfp4_fused_linear_ws(a_codes, a_scales, w_codes, w_scales, M, N, K, segs, nseg, y, ldy,
                               out_dtype, nullptr, 0, stream);
}

nvfp4_status nvfp4_gate_up_silu_quantize(const void* a_codes, const void* a_scales,
                                          const void* w_codes, const void* w_scales, int64_t M,
                                          int64_t H, int64_t K, float a_gs, float w_gs_gate,
                                          float w_gs_up, float h_gs, void* h_codes, void* h_scales,
                                          nvfp4_stream_t stream) {
  if (a_codes == nullptr || a_scales == nullptr || w_codes == nullptr || w_scales == nullptr ||
      h_codes == nullptr || h_scales == nullptr)
    return NVFP4_ERR_INVALID_ARG;
  if (M < 0 || M > kMaxDim || H < 128 || H % 128 != 0 || 2 * H > kMaxDim || K < 64 ||
      K % 64 != 0 || K > kMaxDim)
    return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(a_codes) || !aligned16(a_scales) || !aligned16(w_codes) ||
      !aligned16(w_scales) || !aligned16(h_codes) || !aligned16(h_scales))
    return NVFP4_ERR_ALIGNMENT;
  if (!good_scale(a_gs) || !good_scale(w_gs_gate) || !good_scale(w_gs_up) || !good_scale(h_gs))
    return NVFP4_ERR_INVALID_ARG;
  if (M == 0) return NVFP4_OK;
  int dev;
  DeviceInfo* info;
  nvfp4_status st = current_device(&dev, &info);
  if (st != NVFP4_OK) return st;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);

  nvfp4::GemmArgs g = {};
  g.M = static_cast<int>(M);
  g.N = static_cast<int>(2 * H);
  g.K = static_cast<int>(K);
  g.wait_ns = g_wait_ns;
  g.H = static_cast<int>(H);
  g.alpha_gate = a_gs * w_gs_gate;   // fp32 products, as the segment table forms them
  g.alpha_up = a_gs * w_gs_up;
  g.h_gs = h_gs;
  g.h_codes = static_cast<uint8_t*>(h_codes);
  g.h_scales = static_cast<uint8_t*>(h_scales);
  const int64_t a_bytes = M * (K / 2), w_bytes = 2 * H * (K / 2);
  g.n_fastest = a_bytes > (64ll << 20) && w_bytes < a_bytes;
  nvfp4_segment one = {0, w_gs_gate, a_gs, NVFP4_OP_NONE, nullptr, nullptr};
  SegTable table;
  if ((st = build_segments(&one, 1, 2 * H, &table)) != NVFP4_OK) return st;

  CUtensorMap ta, tb, tsa, tsb;
  if ((st = code_map(a_codes, M, K / 2, nvfp4::tc::BM, dev, &ta)) != NVFP4_OK) return st;
  if ((st = code_map(w_codes, 2 * H, K / 2, nvfp4::tc::BN / 2, dev, &tb)) != NVFP4_OK) return st;
  if ((st = scale_map(a_scales, M, K, 1, dev, &tsa)) != NVFP4_OK) return st;
  if ((st = scale_map(w_scales, 2 * H, K, 1, dev, &tsb)) != NVFP4_OK) return st;

  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[2];
  if ((st = pair_config(nvfp4::k_gemm_tc<2, true>, info, &info->attr_tc2_swiglu,
                        &info->swiglu_pairs, cs, &cfg, attr)) != NVFP4_OK)
    return st;
  const int64_t tiles = ((M + 2 * nvfp4::tc::BM - 1) / (2 * nvfp4::tc::BM)) * (H / 128);
  const int pairs = static_cast<int>(tiles < info->swiglu_pairs ? tiles : info->swiglu_pairs);
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  if (cudaLaunchKernelEx(&cfg, nvfp4::k_gemm_tc<2, true>, ta, tb, tsa, tsb, g, table) !=
      cudaSuccess) {
    cudaGetLastError();
    return NVFP4_ERR_CUDA;
  }
  return check_launch();
}

nvfp4_status nvfp4_linear(const void* a_codes, const void* a_scales, float a_gs,
                          const void* w_codes, const void* w_scales, float w_gs, int64_t M,
                          int64_t N, int64_t K, void* y, int64_t ldy, nvfp4_out_dtype out_dtype,
                          nvfp4_stream_t stream) {
  nvfp4_segment s;
  s.n_offset = 0;
  s.w_gs = w_gs;
  s.a_gs = a_gs;
  s.op = NVFP4_OP_NONE;
  s.a_log = nullptr;
  s.dt_bias = nullptr;
  return nvfp4_fused_linear(a_codes, a_scales, w_codes, w_scales, M, N, K, &s, 1, y, ldy,
                            out_dtype, stream);
}

nvfp4_status nvfp4_silu_mul(const void* gu, int64_t M, int64_t H, int64_t ld_in, void* h,
                            int64_t ld_out, nvfp4_stream_t stream) {
  if (gu == nullptr || h == nullptr) return NVFP4_ERR_INVALID_ARG;
  if (M < 0 || H < 8 || H % 8 != 0 || ld_in < 2 * H || ld_out < H) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(gu) || !aligned16(h) || ld_in % 8 != 0 || ld_out % 8 != 0)
    return NVFP4_ERR_ALIGNMENT;
  if (M == 0) return NVFP4_OK;
  int dev;
  DeviceInfo* info;
  nvfp4_status st = current_device(&dev, &info);
  if (st != NVFP4_OK) return st;
  const int grid = grid_for(M * (H / 8), nvfp4::SILU_THREADS, info->sms * 8);
  nvfp4::k_silu_mul<<<grid, nvfp4::SILU_THREADS, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<const __nv_bfloat16*>(gu), M, H, ld_in, static_cast<__nv_bfloat16*>(h), ld_out);
  return check_launch();
}

float nvfp4_kv_scale(float amax) { return amax > 0.0f ? amax / 448.0f : 1.0f; }

nvfp4_status nvfp4_kv_quantize_fp8(const void* x, int64_t n, float scale, void* out,
                                   nvfp4_stream_t stream) {
  if (x == nullptr || out == nullptr) return NVFP4_ERR_INVALID_ARG;
  if (n < 0 || n % 8 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(x) || !aligned16(out)) return NVFP4_ERR_ALIGNMENT;
  if (!good_scale(scale)) return NVFP4_ERR_INVALID_ARG;
  if (n == 0) return NVFP4_OK;
  int dev;
  DeviceInfo* info;
  nvfp4_status st = current_device(&dev, &info);
  if (st != NVFP4_OK) return st;
  volatile float one = 1.0f;
  const float r = one / scale;   // fp32(1 / scale), IEEE division
  const int grid = grid_for(n / 8, nvfp4::KV_THREADS, info->sms * 8);
  nvfp4::k_kv_fp8<<<grid, nvfp4::KV_THREADS, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<const __nv_bfloat16*>(x), n / 8, r, static_cast<uint2*>(out));
  return check_launch();
}

nvfp4_status nvfp4_gdn_recurrence(const float* q, const float* k, const float* v, const float* g,
                                  const float* beta, int64_t T, int32_t Hv, int32_t group,
                                  int32_t head_dim, float* o, float* state,
                                  nvfp4_stream_t stream) {
  if (q == nullptr || k == nullptr || v == nullptr || g == nullptr || beta == nullptr ||
      o == nullptr || state == nullptr)
    return NVFP4_ERR_INVALID_ARG;
  if (T < 0 || Hv < 1 || group < 1 || Hv % group != 0 || head_dim != nvfp4::gdn::D)
    return NVFP4_ERR_UNSUPPORTED_SHAPE;
  for (const void* p : {static_cast<const void*>(q), static_cast<const void*>(k),
                        static_cast<const void*>(v), static_cast<const void*>(o),
                        static_cast<const void*>(state)})
    if (!aligned16(p)) return NVFP4_ERR_ALIGNMENT;
  int dev;
  DeviceInfo* info;
  nvfp4_status st = current_device(&dev, &info);
  if (st != NVFP4_OK) return st;
  if (!info->attr_gdn) {
    if (cudaFuncSetAttribute(nvfp4::k_gdn_chunked, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             nvfp4::gdn::SMEM_BYTES) != cudaSuccess) {
      cudaGetLastError();
      return NVFP4_ERR_CUDA;
    }
    info->attr_gdn = true;
  }
  nvfp4::GdnArgs a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.g = g;
  a.beta = beta;
  a.o = o;
  a.state = state;
  a.T = T;
  a.Hv = Hv;
  a.group = group;
  // value rows are independent: split each head over enough CTAs to fill the
  // SMs in one wave (at most 8 parts of at least 16 rows)
  int parts = info->sms / Hv;
  if (parts < 1) parts = 1;
  if (parts > 8) parts = 8;
  a.rows = (nvfp4::gdn::D + parts - 1) / parts;
  a.parts = (nvfp4::gdn::D + a.rows - 1) / a.rows;
  nvfp4::k_gdn_chunked<<<Hv * a.parts, nvfp4::gdn::THREADS, nvfp4::gdn::SMEM_BYTES,
                         reinterpret_cast<cudaStream_t>(stream)>>>(a);
  return check_launch();
}

nvfp4_status nvfp4_test_e2m1(const float* in, uint8_t* out, int64_t n, nvfp4_stream_t stream) {
  if (in == nullptr || out == nullptr || n < 0) return NVFP4_ERR_INVALID_ARG;
  if (n == 0) return NVFP4_OK;
  int dev;
  DeviceInfo* info;
  nvfp4_status st = current_device(&dev, &info);
  if (st != NVFP4_OK) return st;
  nvfp4::k_test_e2m1<<<grid_for(n, 256, info->sms * 16), 256, 0,
                       reinterpret_cast<cudaStream_t>(stream)>>>(in, out, n);
  return check_launch();
}

nvfp4_status nvfp4_test_e4m3(const float* in, uint8_t* out, int64_t n, nvfp4_stream_t stream) {
  if (in == nullptr || out == nullptr || n < 0) return NVFP4_ERR_INVALID_ARG;
  if (n == 0) return NVFP4_OK;
  int dev;
  DeviceInfo* info;
  nvfp4_status st = current_device(&dev, &info);
  if (st != NVFP4_OK) return st;
  nvfp4::k_test_e4m3<<<grid_for(n, 256, info->sms * 16), 256, 0,
                       reinterpret_cast<cudaStream_t>(stream)>>>(in, out, n);
  return check_launch();
}

nvfp4_status nvfp4_test_wait_timeout(uint64_t limit_ns, nvfp4_stream_t stream) {
  if (limit_ns == 0) return NVFP4_ERR_INVALID_ARG;
  int dev;
  DeviceInfo* info;
  nvfp4_status st = current_device(&dev, &info);
  if (st != NVFP4_OK) return st;
  nvfp4::k_test_wait_timeout<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(limit_ns);
  if ((st = check_launch()) != NVFP4_OK) return st;
  return nvfp4_last_device_error(stream, nullptr);
}

}  // extern "C"
