// libsbn: C ABI of the Sparse-BitNet BitLinear forward (see include/sbn.h).
//
// Host side of the library: argument validation (before anything touches
// the GPU), device checks, and the launches on the caller's stream. Every
// step of the path runs in the kernels included below; there is no host or
// CPU fallback.

#include "sbn.h"

#include <algorithm>
#include <atomic>
#include <climits>
#include <cstdint>
#include <cstring>
#include <utility>

#include "common.cuh"
#include "qa.cuh"
#include "qw.cuh"
#include "qw_fused.cuh"
#include "qw_stream.cuh"
#include "qw_shard.cuh"
#include "bl_decode.cuh"
#include "bl_decode_res.cuh"
#include "bl_gemv.cuh"
#include "bl_decode_ent.cuh"
#include "expand_dense.cuh"
#include "bl_tc_sp.cuh"
#include "bl_tc2.cuh"
#include "bwd_tc.cuh"
#include "entropy.cuh"
#include "entropy_pack.cuh"
#include "bwd.cuh"
#include "flip.cuh"
#include "bl_tc.cuh"
#include "probe.cuh"

#include <cudaTypedefs.h>

namespace sbn {

namespace {

constexpr int kMaxDevices = 64;
int g_dev_checked[kMaxDevices];  // 0 unknown, 1 ok, -1 unsupported
int g_dev_sms[kMaxDevices];

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0u; }

bool pattern_ok(int n, int m) {
  return (m == 4 || m == 8 || m == 16) && n >= 1 && n <= m && (4 * n) % m == 0;
}

bool prod_lt_2_31(long long a, long long b) { return a >= 0 && b >= 0 && a * b < (1ll << 31); }

size_t round_up16(size_t x) { return (x + 15u) & ~size_t(15); }

// Current device must be an sm_100 part (the library carries sm_100a code only).
sbn_status check_device(int* dev_out, int* sms_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) { cudaGetLastError(); return SBN_ERR_CUDA; }
  if (dev < 0 || dev >= kMaxDevices) return SBN_ERR_DEVICE;
  if (g_dev_checked[dev] == 0) {
    int major = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      return SBN_ERR_CUDA;
    }
    g_dev_sms[dev] = sms;
    g_dev_checked[dev] = (major == 10) ? 1 : -1;
  }
  if (g_dev_checked[dev] < 0) return SBN_ERR_DEVICE;
  *dev_out = dev;
  *sms_out = g_dev_sms[dev];
  return SBN_OK;
}

sbn_status launch_status() {
  return cudaGetLastError() == cudaSuccess ? SBN_OK : SBN_ERR_CUDA;
}

// Programmatic dependent launch of the kernels that call griddep_wait()
// before touching global memory: each may be scheduled while the previous
// grid on the stream is finishing, so its launch and set-up (barriers,
// TMEM, selector tables) overlap that grid's tail. Switched by
// sbn_set_programmatic_launch; on by default.
std::atomic<int> g_pdl{1};

// The dynamic shared-memory limit of a kernel, raised once per device (flags:
// one per device, owned by the caller's instantiation).
template <typename K>
bool set_smem_attr_once(K kern, size_t bytes, bool* flags) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return false;
  }
  if (!flags[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) != cudaSuccess) {
      cudaGetLastError();
      return false;
    }
    flags[dev] = true;
  }
  return true;
}

// cudaLaunchKernelEx with the programmatic attribute (when switched on) and,
// for cluster > 1, clusters of `cluster` CTAs along x.
template <typename... KArgs, typename... Args>
sbn_status launch_ex(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                     unsigned cluster, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  unsigned na = 0;
  if (g_pdl.load(std::memory_order_relaxed)) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  if (cluster > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = cluster;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  if (cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...) != cudaSuccess) {
    cudaGetLastError();
    return SBN_ERR_CUDA;
  }
  return SBN_OK;
}

sbn_status validate_weights_shape(int32_t n_out, int32_t k, int32_t n, int32_t m) {
  if (!pattern_ok(n, m)) return SBN_ERR_PATTERN;
  if (n_out < 1 || k < 128 || (k % 128) != 0) return SBN_ERR_SHAPE;
  if (!prod_lt_2_31(n_out, k)) return SBN_ERR_SHAPE;
  return SBN_OK;
}


// One cooperative launch of qw_stream_kernel: one CTA per SM, so that all
// CTAs are resident for the grid barrier. The bins and the arrival counter
// of the workspace are cleared first, on the same stream.
template <int M>
sbn_status launch_qw_stream(const uint16_t* w, int n_out, int k, int n, uint8_t* codes, int cstride,
                            uint8_t* meta, int mstride, float* gamma, unsigned char* ws, int sms,
                            cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)std::min(sms, kQwMaxGrid));
  cfg.blockDim = dim3(kQsThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, qw_stream_kernel<M>, w, n_out, k, n, codes, cstride, meta, mstride,
                         gamma, ws) != cudaSuccess) {
    cudaGetLastError();
    return SBN_ERR_CUDA;
  }
  return SBN_OK;
}

sbn_status launch_quantize_weights(const uint16_t* w, int n_out, int k, int n, int m, uint8_t* codes,
                                   uint8_t* meta, float* gamma, unsigned char* ws, int sms,
                                   cudaStream_t st) {
  // Each CTA's exact sum counts units of 2^-37 of values below 8 in a u64:
  // at most 2^24 elements per CTA (always true for N_out*K < 2^31 on 128+ SMs).
  if ((long long)n_out * k > ((long long)std::min(sms, kQwMaxGrid) << 24)) return SBN_ERR_SHAPE;
  if (cudaMemsetAsync(ws, 0, kQwClearBytes, st) != cudaSuccess) {
    cudaGetLastError();
    return SBN_ERR_CUDA;
  }
  const int cstride = (int)sbn_codes_row_bytes(k, n, m);
  const int mstride = (int)sbn_meta_row_bytes(k, n, m);
  switch (m) {
    case 4: return launch_qw_stream<4>(w, n_out, k, n, codes, cstride, meta, mstride, gamma, ws, sms, st);
    case 8: return launch_qw_stream<8>(w, n_out, k, n, codes, cstride, meta, mstride, gamma, ws, sms, st);
    default: return launch_qw_stream<16>(w, n_out, k, n, codes, cstride, meta, mstride, gamma, ws, sms, st);
  }
}

template <int MM, int CB, int NT, bool DENSE, bool ACC>
sbn_status launch_decode(const DecodeParams& p, int sms, cudaStream_t st) {
  static bool attr_set = false;  // per instantiation (benign race: same value)
  const size_t smem = decode_smem_bytes(p.rt, NT, CB, DENSE);
  auto kern = bl_decode_kernel<MM, CB, NT, DENSE, ACC>;
  if (!attr_set) {
    // allow the largest footprint this instantiation can be launched with
    const size_t smem_max = decode_smem_bytes(kDecMaxRT, NT, CB, DENSE);
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_max) != cudaSuccess) {
      cudaGetLastError();
      return SBN_ERR_CUDA;
    }
    attr_set = true;
  }
  (void)sms;
  const int rows = 16 * p.rt;
  kern<<<(p.N + rows - 1) / rows, 32 * kDecKS * p.rt, smem, st>>>(p);
  return launch_status();
}

template <int NT, bool ACC>
sbn_status dispatch_decode(const DecodeParams& p, int n, int m, int sms, cudaStream_t st) {
  const int cb = 4 * n / m;
  if (n == m) return launch_decode<8, 4, NT, true, ACC>(p, sms, st);
  switch (m * 8 + cb) {
    case 4 * 8 + 1: return launch_decode<4, 1, NT, false, ACC>(p, sms, st);
    case 4 * 8 + 2: return launch_decode<4, 2, NT, false, ACC>(p, sms, st);
    case 4 * 8 + 3: return launch_decode<4, 3, NT, false, ACC>(p, sms, st);
    case 8 * 8 + 1: return launch_decode<8, 1, NT, false, ACC>(p, sms, st);
    case 8 * 8 + 2: return launch_decode<8, 2, NT, false, ACC>(p, sms, st);
    case 8 * 8 + 3: return launch_decode<8, 3, NT, false, ACC>(p, sms, st);
    case 16 * 8 + 1: return launch_decode<16, 1, NT, false, ACC>(p, sms, st);
    case 16 * 8 + 2: return launch_decode<16, 2, NT, false, ACC>(p, sms, st);
    case 16 * 8 + 3: return launch_decode<16, 3, NT, false, ACC>(p, sms, st);
  }
  return SBN_ERR_PATTERN;
}

// Resident decode kernel: grid = min(SMs, tiles), one CTA per SM holding the
// packed rows of its tiles and all of Xq in shared memory.
template <int MM, int CB, int NT, bool DENSE, bool ACC, bool XBF>
sbn_status launch_decode_res(const DresParams& p, int grid, size_t smem, cudaStream_t st) {
  static bool attr_set[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return SBN_ERR_CUDA;
  }
  auto kern = bl_decode_res_kernel<MM, CB, NT, DENSE, ACC, XBF>;
  if (!attr_set[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kDresSmemMax) !=
        cudaSuccess) {
      cudaGetLastError();
      return SBN_ERR_CUDA;
    }
    attr_set[dev] = true;
  }
  kern<<<grid, kDresThreads, smem, st>>>(p);
  return launch_status();
}

template <int NT, bool ACC, bool XBF>
sbn_status dispatch_decode_res(const DresParams& p, int n, int m, int grid, size_t smem,
                               cudaStream_t st) {
  const int cb = 4 * n / m;
  if (n == m) return launch_decode_res<8, 4, NT, true, ACC, XBF>(p, grid, smem, st);
  switch (m * 8 + cb) {
    case 4 * 8 + 1: return launch_decode_res<4, 1, NT, false, ACC, XBF>(p, grid, smem, st);
    case 4 * 8 + 2: return launch_decode_res<4, 2, NT, false, ACC, XBF>(p, grid, smem, st);
    case 4 * 8 + 3: return launch_decode_res<4, 3, NT, false, ACC, XBF>(p, grid, smem, st);
    case 8 * 8 + 1: return launch_decode_res<8, 1, NT, false, ACC, XBF>(p, grid, smem, st);
    case 8 * 8 + 2: return launch_decode_res<8, 2, NT, false, ACC, XBF>(p, grid, smem, st);
    case 8 * 8 + 3: return launch_decode_res<8, 3, NT, false, ACC, XBF>(p, grid, smem, st);
    case 16 * 8 + 1: return launch_decode_res<16, 1, NT, false, ACC, XBF>(p, grid, smem, st);
    case 16 * 8 + 2: return launch_decode_res<16, 2, NT, false, ACC, XBF>(p, grid, smem, st);
    case 16 * 8 + 3: return launch_decode_res<16, 3, NT, false, ACC, XBF>(p, grid, smem, st);
  }
  return SBN_ERR_PATTERN;
}

// Decode GEMV (T <= 16): one CTA per SM, launched with programmatic
// dependent launch so that its launch overlaps the tail of the previous
// kernel on the stream (the kernel waits for that grid before it reads).
template <int MM, int CB, int NT, bool DENSE, bool ACC, bool XBF>
sbn_status launch_gemv(const GvParams& p, int grid, size_t smem, cudaStream_t st) {
  static bool attr_set[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return SBN_ERR_CUDA;
  }
  auto kern = bl_gemv_kernel<MM, CB, NT, DENSE, ACC, XBF>;
  if (!attr_set[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGvSmemMax) !=
        cudaSuccess) {
      cudaGetLastError();
      return SBN_ERR_CUDA;
    }
    attr_set[dev] = true;
  }
  return launch_ex(kern, dim3((unsigned)grid), dim3(kGvThreads), smem, st, 1, p);
}

template <int NT, bool ACC, bool XBF>
sbn_status dispatch_gemv(const GvParams& p, int n, int m, int grid, size_t smem, cudaStream_t st) {
  const int cb = 4 * n / m;
  if (n == m) return launch_gemv<8, 4, NT, true, ACC, XBF>(p, grid, smem, st);
  switch (m * 8 + cb) {
    case 4 * 8 + 1: return launch_gemv<4, 1, NT, false, ACC, XBF>(p, grid, smem, st);
    case 4 * 8 + 2: return launch_gemv<4, 2, NT, false, ACC, XBF>(p, grid, smem, st);
    case 4 * 8 + 3: return launch_gemv<4, 3, NT, false, ACC, XBF>(p, grid, smem, st);
    case 8 * 8 + 1: return launch_gemv<8, 1, NT, false, ACC, XBF>(p, grid, smem, st);
    case 8 * 8 + 2: return launch_gemv<8, 2, NT, false, ACC, XBF>(p, grid, smem, st);
    case 8 * 8 + 3: return launch_gemv<8, 3, NT, false, ACC, XBF>(p, grid, smem, st);
    case 16 * 8 + 1: return launch_gemv<16, 1, NT, false, ACC, XBF>(p, grid, smem, st);
    case 16 * 8 + 2: return launch_gemv<16, 2, NT, false, ACC, XBF>(p, grid, smem, st);
    case 16 * 8 + 3: return launch_gemv<16, 3, NT, false, ACC, XBF>(p, grid, smem, st);
  }
  return SBN_ERR_PATTERN;
}

// Grid, CTA range and shared memory of the decode GEMV; false when the shape
// is outside it (t > 16, activation rows beyond the registers' reach, or
// rows that do not fit in shared memory).
bool gemv_fits(int32_t t, int32_t k, int32_t n_out, int32_t n, int32_t m, int sms, bool xbf, int* grid,
               int* per_cta, size_t* smem) {
  if (t < 1 || t > 16) return false;
  // the consumer threads hold every activation chunk in registers
  const long long chunks = (long long)t * (xbf ? k / 8 : k / 16);
  if (chunks > (long long)kGvConsumers * kGvMaxChunks) return false;
  const int cstride = (int)sbn_codes_row_bytes(k, n, m);
  const int mstride = (int)sbn_meta_row_bytes(k, n, m);
  const int tiles = (n_out + 15) / 16;
  *grid = std::min(sms, tiles);
  *per_cta = (tiles + *grid - 1) / *grid;
  const GvLayout L = gv_layout(*per_cta, t <= 8 ? 8 : 16, t, k, cstride, mstride, n == m);
  *smem = L.total;
  return *per_cta <= kGvMaxTiles && L.total <= kGvSmemMax;
}

// One launch of the decode GEMV. XBF: bf16 activations xbf, quantized in the
// kernel (optional copies to xq_out, xs_out); else xq, xs.
template <bool ACC, bool XBF>
sbn_status run_gemv(const int8_t* xq, const float* xs, const uint16_t* xbf, int8_t* xq_out, float* xs_out,
                    int32_t t, int32_t k, int32_t n_out, int32_t n, int32_t m, const uint8_t* codes,
                    const uint8_t* meta, const float* gamma, uint16_t* y, int32_t* acc, int grid, int per_cta,
                    size_t smem, cudaStream_t cs) {
  GvParams q;
  q.xq = xq; q.xs = xs; q.xbf = xbf; q.xq_out = xq_out; q.xs_out = xs_out;
  q.codes = codes; q.meta = meta; q.gamma = gamma; q.y = y; q.acc_out = acc;
  q.T = t; q.K = k; q.N = n_out;
  q.cstride = (int)sbn_codes_row_bytes(k, n, m); q.mstride = (int)sbn_meta_row_bytes(k, n, m);
  q.tiles_per_cta = per_cta;
  const int tiles = (n_out + 15) / 16;
  q.tile_base = tiles / grid;
  q.tile_rem = tiles % grid;
  q.L = gv_layout(per_cta, t <= 8 ? 8 : 16, t, k, q.cstride, q.mstride, n == m);
  q.kc = XBF ? k / 8 : k / 16;
  q.kc_magic = (uint32_t)(((1ull << 32) + (unsigned long long)q.kc - 1) / (unsigned long long)q.kc);
  q.dr = kGvConsumers / q.kc;
  q.drem = kGvConsumers % q.kc;
  return t <= 8 ? dispatch_gemv<8, ACC, XBF>(q, n, m, grid, smem, cs)
                : dispatch_gemv<16, ACC, XBF>(q, n, m, grid, smem, cs);
}

// Decode contraction over entropy-tight weights (patterns with m = 4 or 8).
template <int MM, int CB, int NT, bool ACC, bool XBF>
sbn_status launch_decode_ent(const DresParams& p, int grid, size_t smem, cudaStream_t st) {
  static bool attr_set[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return SBN_ERR_CUDA;
  }
  auto kern = bl_decode_ent_kernel<MM, CB, NT, ACC, XBF>;
  if (!attr_set[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kDresSmemMax) !=
        cudaSuccess) {
      cudaGetLastError();
      return SBN_ERR_CUDA;
    }
    attr_set[dev] = true;
  }
  kern<<<grid, kDresThreads, smem, st>>>(p);
  return launch_status();
}

template <int NT, bool ACC, bool XBF>
sbn_status dispatch_decode_ent(const DresParams& p, int n, int m, int grid, size_t smem,
                               cudaStream_t st) {
  switch (m * 8 + 4 * n / m) {
    case 4 * 8 + 1: return launch_decode_ent<4, 1, NT, ACC, XBF>(p, grid, smem, st);
    case 4 * 8 + 2: return launch_decode_ent<4, 2, NT, ACC, XBF>(p, grid, smem, st);
    case 4 * 8 + 3: return launch_decode_ent<4, 3, NT, ACC, XBF>(p, grid, smem, st);
    case 8 * 8 + 1: return launch_decode_ent<8, 1, NT, ACC, XBF>(p, grid, smem, st);
    case 8 * 8 + 2: return launch_decode_ent<8, 2, NT, ACC, XBF>(p, grid, smem, st);
    case 8 * 8 + 3: return launch_decode_ent<8, 3, NT, ACC, XBF>(p, grid, smem, st);
  }
  return SBN_ERR_PATTERN;
}

// cuTensorMapEncodeTiled from the driver, looked up once (no libcuda link).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

template <int MM, int CB, bool DENSE, bool ACC>
sbn_status launch_tc(const CUtensorMap& tm, const TcParams& p, int sms, cudaStream_t st) {
  static bool attr_set[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return SBN_ERR_CUDA;
  }
  auto kern = bl_tc_kernel<MM, CB, DENSE, ACC>;
  if (!attr_set[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kTcSmemBytes) !=
        cudaSuccess) {
      cudaGetLastError();
      return SBN_ERR_CUDA;
    }
    attr_set[dev] = true;
  }
  const int tiles = ((p.N + kTcBM - 1) / kTcBM) * ((p.T + kTcBN - 1) / kTcBN);
  kern<<<std::min(tiles, sms), kTcThreads, kTcSmemBytes, st>>>(tm, p);
  return launch_status();
}

// Packed weights, expanded in the kernel (no workspace).
template <bool ACC>
sbn_status dispatch_tc(const CUtensorMap& tm, const TcParams& p, int n, int m, int sms, cudaStream_t st) {
  const int cb = 4 * n / m;
  if (n == m) return launch_tc<8, 4, true, ACC>(tm, p, sms, st);
  switch (m * 8 + cb) {
    case 4 * 8 + 1: return launch_tc<4, 1, false, ACC>(tm, p, sms, st);
    case 4 * 8 + 2: return launch_tc<4, 2, false, ACC>(tm, p, sms, st);
    case 4 * 8 + 3: return launch_tc<4, 3, false, ACC>(tm, p, sms, st);
    case 8 * 8 + 1: return launch_tc<8, 1, false, ACC>(tm, p, sms, st);
    case 8 * 8 + 2: return launch_tc<8, 2, false, ACC>(tm, p, sms, st);
    case 8 * 8 + 3: return launch_tc<8, 3, false, ACC>(tm, p, sms, st);
    case 16 * 8 + 1: return launch_tc<16, 1, false, ACC>(tm, p, sms, st);
    case 16 * 8 + 2: return launch_tc<16, 2, false, ACC>(tm, p, sms, st);
    case 16 * 8 + 3: return launch_tc<16, 3, false, ACC>(tm, p, sms, st);
  }
  return SBN_ERR_PATTERN;
}

// Expansion of the packed weights into the dense int8 workspace [N_out, K].
template <int MM, int CB, bool DENSE>
sbn_status launch_expand(const uint8_t* codes, const uint8_t* meta, int n_out, int k, int cstride,
                         int mstride, int8_t* wd, int sms, cudaStream_t st) {
  const long long chunks = ((long long)n_out * (k / 16) + 31) / 32;
  const int grid = (int)std::max(1LL, std::min(chunks, (long long)sms * 4));
  return launch_ex(expand_dense_kernel<MM, CB, DENSE>, dim3(grid), dim3(kXdThreads), 0, st, 1, codes, meta, n_out, k,
                   cstride, mstride, wd);
}

sbn_status dispatch_expand(const uint8_t* codes, const uint8_t* meta, int n_out, int k, int n, int m,
                           int cstride, int mstride, int8_t* wd, int sms, cudaStream_t st) {
  const int cb = 4 * n / m;
  if (n == m) return launch_expand<8, 4, true>(codes, meta, n_out, k, cstride, mstride, wd, sms, st);
  switch (m * 8 + cb) {
    case 4 * 8 + 1: return launch_expand<4, 1, false>(codes, meta, n_out, k, cstride, mstride, wd, sms, st);
    case 4 * 8 + 2: return launch_expand<4, 2, false>(codes, meta, n_out, k, cstride, mstride, wd, sms, st);
    case 4 * 8 + 3: return launch_expand<4, 3, false>(codes, meta, n_out, k, cstride, mstride, wd, sms, st);
    case 8 * 8 + 1: return launch_expand<8, 1, false>(codes, meta, n_out, k, cstride, mstride, wd, sms, st);
    case 8 * 8 + 2: return launch_expand<8, 2, false>(codes, meta, n_out, k, cstride, mstride, wd, sms, st);
    case 8 * 8 + 3: return launch_expand<8, 3, false>(codes, meta, n_out, k, cstride, mstride, wd, sms, st);
    case 16 * 8 + 1: return launch_expand<16, 1, false>(codes, meta, n_out, k, cstride, mstride, wd, sms, st);
    case 16 * 8 + 2: return launch_expand<16, 2, false>(codes, meta, n_out, k, cstride, mstride, wd, sms, st);
    case 16 * 8 + 3: return launch_expand<16, 3, false>(codes, meta, n_out, k, cstride, mstride, wd, sms, st);
  }
  return SBN_ERR_PATTERN;
}

// TMA map of the INT8 activations [T, K]: boxes of box_rows tokens x 128
// bytes, 128-byte swizzle (the layout the MMA descriptors describe).
sbn_status make_act_tensor_map(CUtensorMap* tm, const int8_t* xq, int t, int k, int box_rows = kTcBN) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return SBN_ERR_CUDA;
  cuuint64_t gdim[2] = {(cuuint64_t)k, (cuuint64_t)t};
  cuuint64_t gstride[1] = {(cuuint64_t)k};
  cuuint32_t box[2] = {(cuuint32_t)kTcBK, (cuuint32_t)box_rows};
  cuuint32_t estride[2] = {1, 1};
  const CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t*>(xq), gdim, gstride, box,
                         estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? SBN_OK : SBN_ERR_CUDA;
}

// TMA map of the expanded int8 weights [N_out, K]: boxes of 128 rows x 128
// bytes, 128-byte swizzle (the layout the A descriptor describes).
sbn_status make_weight_tensor_map(CUtensorMap* tm, const int8_t* wd, int n_out, int k) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return SBN_ERR_CUDA;
  cuuint64_t gdim[2] = {(cuuint64_t)k, (cuuint64_t)n_out};
  cuuint64_t gstride[1] = {(cuuint64_t)k};
  cuuint32_t box[2] = {(cuuint32_t)kTcBK, (cuuint32_t)kTcBM};
  cuuint32_t estride[2] = {1, 1};
  const CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t*>(wd), gdim, gstride, box,
                         estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? SBN_OK : SBN_ERR_CUDA;
}

// TMA maps of the compressed 2:4 workspace: kept values [N_out, K/2] in
// boxes of 128 rows x 128 bytes (128-byte swizzle), metadata [N_pad, K/8] in
// boxes of 128 rows x 16 bytes (no swizzle).
sbn_status make_sp_weight_maps(CUtensorMap* tw, CUtensorMap* te, const int8_t* wsp, const uint8_t* esp,
                               int n_out, int n_pad, int k) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return SBN_ERR_CUDA;
  cuuint32_t estride[2] = {1, 1};
  cuuint64_t wdim[2] = {(cuuint64_t)(k / 2), (cuuint64_t)n_out};
  cuuint64_t wstr[1] = {(cuuint64_t)(k / 2)};
  cuuint32_t wbox[2] = {128, (cuuint32_t)kSpBM};
  CUresult r = enc(tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t*>(wsp), wdim, wstr, wbox, estride,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return SBN_ERR_CUDA;
  cuuint64_t edim[2] = {(cuuint64_t)(k / 8), (cuuint64_t)n_pad};
  cuuint64_t estr[1] = {(cuuint64_t)(k / 8)};
  cuuint32_t ebox[2] = {(cuuint32_t)(kSpBK / 8), (cuuint32_t)kSpBM};
  r = enc(te, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(esp), edim, estr, ebox, estride,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? SBN_OK : SBN_ERR_CUDA;
}

// Compressed 2:4 workspace: kept values [N_out, K/2], then (at a 128-byte
// boundary) the metadata [N_pad, K/8], N_pad = N_out rounded up to 256 (the
// rows of a CTA pair's tile; pad rows carry valid metadata).
constexpr int kSpRowPad = 256;
int sp_rows_padded(int32_t n_out) { return (n_out + kSpRowPad - 1) / kSpRowPad * kSpRowPad; }
size_t sp_values_bytes(int32_t k, int32_t n_out) {
  return ((size_t)n_out * (size_t)(k / 2) + 127) & ~(size_t)127;
}
size_t sp_ws_bytes(int32_t k, int32_t n_out) {
  return sp_values_bytes(k, n_out) + (size_t)sp_rows_padded(n_out) * (size_t)(k / 8);
}

// Bytes of the optional workspace of the contraction when t selects the
// tensor-core kernel: room for the dense int8 expansion and for the
// compressed 2:4 form, whichever is larger; else none.
size_t bitlinear_ws_bytes(int32_t t, int32_t k, int32_t n_out) {
  return t > 16 ? std::max((size_t)n_out * (size_t)k, sp_ws_bytes(k, n_out)) : 0;
}

template <bool ACC>
sbn_status launch_tc_sp(const CUtensorMap& tm, const TcParams& p, int sms, cudaStream_t st) {
  static bool attr_set[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return SBN_ERR_CUDA;
  }
  auto kern = bl_tc_sp_kernel<ACC>;
  if (!attr_set[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSpSmemBytes) !=
        cudaSuccess) {
      cudaGetLastError();
      return SBN_ERR_CUDA;
    }
    attr_set[dev] = true;
  }
  const int tiles = ((p.N + kSpBM - 1) / kSpBM) * ((p.T + kSpBN - 1) / kSpBN);
  kern<<<std::min(tiles, sms), kTcThreads, kSpSmemBytes, st>>>(tm, p);
  return launch_status();
}

// CTA pairs of the pair kernel that can be resident at once on this device
// (clusters of two need both SMs in one GPC); 0 if none.
template <bool SPARSE, bool ACC, bool NARROW = false>
int tc2_max_pairs() {
  static int cached[kMaxDevices];   // 0 unknown, else pairs + 1
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return 0;
  }
  if (cached[dev] == 0) {
    using C = T2Cfg<SPARSE, NARROW>;
    auto kern = bl_tc2_kernel<SPARSE, ACC, NARROW>;
    int pairs = 0;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM) == cudaSuccess) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(2);
      cfg.blockDim = dim3(kT2Threads);
      cfg.dynamicSmemBytes = C::SMEM;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      if (cudaOccupancyMaxActiveClusters(&pairs, kern, &cfg) != cudaSuccess) pairs = 0;
    }
    cudaGetLastError();
    cached[dev] = pairs + 1;
  }
  return cached[dev] - 1;
}

// TMA map of the bf16 output [T, N_out] for the pair kernel's tile stores:
// boxes of 32 tokens x 32 rows.
bool make_out_tensor_map(CUtensorMap* ty, const uint16_t* y, int t, int n_out) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t gdim[2] = {(cuuint64_t)n_out, (cuuint64_t)t};
  cuuint64_t gstride[1] = {(cuuint64_t)n_out * 2};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t estride[2] = {1, 1};
  return enc(ty, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(y), gdim, gstride, box, estride,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool SPARSE, bool ACC, bool NARROW = false>
sbn_status launch_tc2(const CUtensorMap& tm, const CUtensorMap& tw, const CUtensorMap& te, const TcParams& p,
                      int max_pairs, cudaStream_t st) {
  using C = T2Cfg<SPARSE, NARROW>;
  // tile stores of the output where every row starts on a 16-byte boundary
  const bool al = !ACC && p.y && (p.N % 8) == 0 && (reinterpret_cast<uintptr_t>(p.y) & 15u) == 0;
  CUtensorMap ty = tm;   // unused unless y_tma
  const int y_tma = (al && make_out_tensor_map(&ty, p.y, p.T, p.N)) ? 1 : 0;
  const int tiles = ((p.N + 255) / 256) * ((p.T + C::BN - 1) / C::BN);
  return launch_ex(bl_tc2_kernel<SPARSE, ACC, NARROW>, dim3(2 * std::min(tiles, max_pairs)), dim3(kT2Threads), C::SMEM,
                   st, 2, tm, tw, te, ty, p, y_tma);
}

// Whether the dense pair kernel should take 128-token tiles: waves of tiles
// over the resident pairs, a narrow tile (half the MMA work, the same
// per-stage cost in the MMA thread) counted as 0.6 of a 256-token one. The
// narrow tiles win where the wide ones leave pairs idle (few tiles, or a
// short last wave).
bool tc2_narrow_pays(int t, int n_out, int wide_pairs, int narrow_pairs) {
  if (narrow_pairs <= 0) return false;
  const long long rp = (n_out + 255) / 256;
  const long long wide = rp * ((t + 255) / 256), narrow = rp * ((t + 127) / 128);
  const long long rw = (wide + wide_pairs - 1) / wide_pairs, rn = (narrow + narrow_pairs - 1) / narrow_pairs;
  return 6 * rn < 10 * rw;
}

// 2:4 weights on the sparse tensor-core MMA: expanded once into the
// compressed workspace for the CTA-pair kernel (ws non-NULL and pairs can
// be resident), else inside the single-CTA kernel.
template <bool ACC_OUT>
sbn_status run_bitlinear_sp(const int8_t* xq, const TcParams& p, void* ws, int sms, cudaStream_t st) {
  CUtensorMap tm;
  sbn_status s2;
  const int pairs = ws ? tc2_max_pairs<true, ACC_OUT>() : 0;
  if (pairs <= 0) {
    if ((s2 = make_act_tensor_map(&tm, xq, p.T, p.K, kSpBN)) != SBN_OK) return s2;
    return launch_tc_sp<ACC_OUT>(tm, p, sms, st);
  }
  const int n_pad = sp_rows_padded(p.N);
  int8_t* wsp = reinterpret_cast<int8_t*>(ws);
  uint8_t* esp = reinterpret_cast<uint8_t*>(ws) + sp_values_bytes(p.K, p.N);
  static bool attr_set[kMaxDevices] = {};
  if (!set_smem_attr_once(expand_sparse24_kernel, kSpXExclusiveSmem, attr_set)) return SBN_ERR_CUDA;
  const long long groups = (long long)n_pad * (p.K / 128);
  const int grid = (int)std::max(1LL, std::min((groups + 31) / 32, (long long)sms));
  if ((s2 = launch_ex(expand_sparse24_kernel, dim3(grid), dim3(kSpXThreads), kSpXExclusiveSmem, st, 1, p.codes,
                      p.meta, p.N, n_pad, p.K, p.cstride, p.mstride, wsp, esp)) != SBN_OK)
    return s2;
  CUtensorMap tw, te;
  if ((s2 = make_sp_weight_maps(&tw, &te, wsp, esp, p.N, n_pad, p.K)) != SBN_OK) return s2;
  if ((s2 = make_act_tensor_map(&tm, xq, p.T, p.K, T2Cfg<true>::HALF)) != SBN_OK) return s2;
  return launch_tc2<true, ACC_OUT>(tm, tw, te, p, pairs, st);
}

template <bool ACC_OUT>
sbn_status run_bitlinear(const int8_t* xq, const float* xs, int32_t t, int32_t k, int32_t n_out,
                         int32_t n, int32_t m, const uint8_t* codes, const uint8_t* meta,
                         const float* gamma, uint16_t* y, int32_t* acc, void* ws, int sms,
                         cudaStream_t st) {
  const int cstride = (int)sbn_codes_row_bytes(k, n, m);
  const int mstride = (int)sbn_meta_row_bytes(k, n, m);
  if (t <= 16) {
    int ggrid = 0, gper = 0;
    size_t gsmem = 0;
    if (gemv_fits(t, k, n_out, n, m, sms, false, &ggrid, &gper, &gsmem))
      return run_gemv<ACC_OUT, false>(xq, xs, nullptr, nullptr, nullptr, t, k, n_out, n, m, codes, meta, gamma,
                                      y, acc, ggrid, gper, gsmem, st);
    // resident kernel when the largest CTA's rows and Xq fit in shared memory
    const int tiles = (n_out + 15) / 16;
    const int grid = std::min(sms, tiles);
    const int per_cta = (tiles + grid - 1) / grid;
    const int nt = t <= 8 ? 8 : 16;
    const DresLayout L = dres_layout(per_cta, nt, k, cstride, mstride, n == m);
    if (per_cta <= kDresMaxTiles && L.total <= kDresSmemMax) {
      DresParams q;
      q.xq = xq; q.xs = xs; q.codes = codes; q.meta = meta; q.gamma = gamma; q.y = y; q.acc_out = acc;
      q.T = t; q.K = k; q.N = n_out; q.cstride = cstride; q.mstride = mstride; q.tiles_per_cta = per_cta;
      q.xbf = nullptr; q.xq_out = nullptr; q.xs_out = nullptr;
      return t <= 8 ? dispatch_decode_res<8, ACC_OUT, false>(q, n, m, grid, L.total, st)
                    : dispatch_decode_res<16, ACC_OUT, false>(q, n, m, grid, L.total, st);
    }
    DecodeParams p;
    p.xq = xq; p.xs = xs; p.codes = codes; p.meta = meta; p.gamma = gamma; p.y = y; p.acc_out = acc;
    p.T = t; p.K = k; p.N = n_out; p.cstride = cstride; p.mstride = mstride;
    p.rt = std::min(kDecMaxRT, std::max(1, (tiles + sms - 1) / sms));
    return t <= 8 ? dispatch_decode<8, ACC_OUT>(p, n, m, sms, st)
                  : dispatch_decode<16, ACC_OUT>(p, n, m, sms, st);
  }
  TcParams p;
  p.codes = codes; p.meta = meta; p.xs = xs; p.gamma = gamma; p.y = y; p.acc_out = acc;
  p.T = t; p.K = k; p.N = n_out; p.cstride = cstride; p.mstride = mstride;
  if (n == 2 && m == 4) return run_bitlinear_sp<ACC_OUT>(xq, p, ws, sms, st);
  CUtensorMap tm;
  const int pairs = ws ? tc2_max_pairs<false, ACC_OUT>() : 0;
  if (pairs > 0) {
    // expand once into the workspace, then TMA both operands on CTA pairs
    int8_t* wd = reinterpret_cast<int8_t*>(ws);
    sbn_status s2 = dispatch_expand(codes, meta, n_out, k, n, m, cstride, mstride, wd, sms, st);
    if (s2 != SBN_OK) return s2;
    CUtensorMap tw;
    if ((s2 = make_weight_tensor_map(&tw, wd, n_out, k)) != SBN_OK) return s2;
    const int npairs = tc2_max_pairs<false, ACC_OUT, true>();
    if (tc2_narrow_pays(t, n_out, pairs, npairs)) {
      if ((s2 = make_act_tensor_map(&tm, xq, t, k, T2Cfg<false, true>::HALF)) != SBN_OK) return s2;
      return launch_tc2<false, ACC_OUT, true>(tm, tw, tw, p, npairs, st);
    }
    if ((s2 = make_act_tensor_map(&tm, xq, t, k, T2Cfg<false>::HALF)) != SBN_OK) return s2;
    return launch_tc2<false, ACC_OUT>(tm, tw, tw, p, pairs, st);
  }
  const sbn_status st_map = make_act_tensor_map(&tm, xq, t, k);
  if (st_map != SBN_OK) return st_map;
  return dispatch_tc<ACC_OUT>(tm, p, n, m, sms, st);
}

// The workspace argument of the contraction: NULL (no expansion buffer), or
// 16-byte aligned and at least bitlinear_ws_bytes long. Unused (NULL) for t <= 16.
sbn_status check_bitlinear_ws(int32_t t, int32_t k, int32_t n_out, void*& ws, size_t ws_bytes) {
  if (!ws) return SBN_OK;
  const size_t need = bitlinear_ws_bytes(t, k, n_out);
  if (need == 0) {
    ws = nullptr;
    return SBN_OK;
  }
  if (!aligned16(ws)) return SBN_ERR_ALIGN;
  if (ws_bytes < need) return SBN_ERR_WORKSPACE;
  return SBN_OK;
}

sbn_status validate_bitlinear(const int8_t* xq, int32_t t, int32_t k, int32_t n_out, int32_t n,
                              int32_t m, const uint8_t* codes, const uint8_t* meta) {
  if (!xq || !codes || (n != m && !meta)) return SBN_ERR_NULL;
  if (!pattern_ok(n, m)) return SBN_ERR_PATTERN;
  if (t < 1 || n_out < 1 || k < 128 || (k % 128) != 0) return SBN_ERR_SHAPE;
  if (!prod_lt_2_31(t, k) || !prod_lt_2_31(n_out, k) || !prod_lt_2_31(t, n_out)) return SBN_ERR_SHAPE;
  if (!aligned16(xq) || !aligned16(codes) || (meta && !aligned16(meta))) return SBN_ERR_ALIGN;
  return SBN_OK;
}

// Fused decode (activation quantization inside the contraction): used when
// t <= 16 and the layout with the bf16 activations fits in shared memory.
bool fused_decode_fits(int32_t t, int32_t k, int32_t n_out, int32_t n, int32_t m, int sms, int* grid,
                       int* per_cta, size_t* smem) {
  if (t > 16) return false;
  const int cstride = (int)sbn_codes_row_bytes(k, n, m);
  const int mstride = (int)sbn_meta_row_bytes(k, n, m);
  const int tiles = (n_out + 15) / 16;
  *grid = std::min(sms, tiles);
  *per_cta = (tiles + *grid - 1) / *grid;
  const DresLayout L = dres_layout(*per_cta, t <= 8 ? 8 : 16, k, cstride, mstride, n == m, true);
  *smem = L.total;
  return *per_cta <= kDresMaxTiles && L.total <= kDresSmemMax;
}

// Workspace of sbn_bitlinear_x when it runs as two steps: Xq and s, then
// the contraction's own workspace (the same size whatever the device).
size_t bitlinear_x_ws_bytes(int32_t t, int32_t k, int32_t n_out) {
  return round_up16((size_t)t * k) + round_up16((size_t)t * 4) + bitlinear_ws_bytes(t, k, n_out);
}

// CTAs of `kern` (threads per CTA, no dynamic shared memory) resident per SM,
// cached per device in `cache` (one slot per device, owned by the caller's
// instantiation); 1 if the query fails.
template <typename K>
int resident_ctas(K kern, int threads, int* cache) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return 1;
  }
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, threads, 0) != cudaSuccess || n < 1) n = 1;
    cudaGetLastError();
    cache[dev] = n;
  }
  return cache[dev];
}

// A quantize_acts kernel over a full wave of CTAs (at most one per token row);
// the residency cache is per kernel (the template argument).
template <auto KERN>
sbn_status launch_qa(int threads, int t, int sms, cudaStream_t s, const uint4* x, int kc, uint2* q, float* x_scale) {
  static int cache[kMaxDevices];
  const long long wave = (long long)resident_ctas(KERN, threads, cache) * sms;
  const int grid = (int)std::max(1LL, std::min(wave, (long long)t));
  return launch_ex(KERN, dim3(grid), dim3(threads), 0, s, 1, x, t, kc, q, x_scale);
}

// One warp per token row up to K = 2560, else one CTA per row (qa.cuh); rows
// up to 16 * 128 * 8 positions stay in registers.
sbn_status launch_quantize_acts(const void* x_bf16, int t, int k, int8_t* xq, float* x_scale, int sms,
                                cudaStream_t s) {
  const int kc = k / 8;
  const uint4* x = reinterpret_cast<const uint4*>(x_bf16);
  uint2* q = reinterpret_cast<uint2*>(xq);
  if (kc <= 32 * 4) return launch_qa<qa_warp_kernel<4>>(kQawThreads, t, sms, s, x, kc, q, x_scale);
  if (kc <= 32 * 8) return launch_qa<qa_warp_kernel<8>>(kQawThreads, t, sms, s, x, kc, q, x_scale);
  if (kc <= 32 * 10) return launch_qa<qa_warp_kernel<10>>(kQawThreads, t, sms, s, x, kc, q, x_scale);
  const int need = (kc + kQaThreads - 1) / kQaThreads;   // >= 3 here
  if (need <= 4) return launch_qa<qa_kernel<4>>(kQaThreads, t, sms, s, x, kc, q, x_scale);
  if (need <= 8) return launch_qa<qa_kernel<8>>(kQaThreads, t, sms, s, x, kc, q, x_scale);
  if (need <= 12) return launch_qa<qa_kernel<12>>(kQaThreads, t, sms, s, x, kc, q, x_scale);
  if (need <= 16) return launch_qa<qa_kernel<16>>(kQaThreads, t, sms, s, x, kc, q, x_scale);
  return launch_qa<qa_kernel_long>(kQaThreads, t, sms, s, x, kc, q, x_scale);
}

// Grid, CTA range and shared memory of the entropy decode; false when the
// shape is outside it (t > 16, or rows that do not fit in shared memory).
bool ent_decode_fits(int32_t t, int32_t k, int32_t n_out, int32_t n, int32_t m, int sms, bool xbf,
                     int* grid, int* per_cta, size_t* smem) {
  if (t < 1 || t > 16) return false;
  const int estride = (int)entropy_row_bytes(k, n, m);
  const int tiles = (n_out + 15) / 16;
  *grid = std::min(sms, tiles);
  *per_cta = (tiles + *grid - 1) / *grid;
  const DresLayout L = dres_layout(*per_cta, t <= 8 ? 8 : 16, k, estride, 0, true, xbf);
  *smem = ent_smem_bytes(L);
  return *per_cta <= kDresMaxTiles && *smem <= kDresSmemMax;
}

sbn_status ent_decode_args(int32_t t, int32_t k, int32_t n_out, int32_t n, int32_t m) {
  if (!pattern_ok(n, m)) return SBN_ERR_PATTERN;
  if (n == m || (m != 4 && m != 8)) return SBN_ERR_PATTERN;
  if (t < 1 || t > 16 || n_out < 1 || k < 128 || (k % 128) != 0 || !prod_lt_2_31(n_out, k))
    return SBN_ERR_SHAPE;
  return SBN_OK;
}

// One launch of the entropy decode. XBF: bf16 activations xbf, quantized in
// the kernel (optional copies to xq_out, xs_out); else xq, xs.
template <bool ACC, bool XBF>
sbn_status launch_bitlinear_entropy(const int8_t* xq, const float* xs, const uint16_t* xbf, int8_t* xq_out,
                                    float* xs_out, int32_t t, int32_t k, int32_t n_out, int32_t n,
                                    int32_t m, const uint8_t* ent, const float* gamma, uint16_t* y,
                                    int32_t* acc, int grid, int per_cta, size_t smem, cudaStream_t cs) {
  DresParams q;
  q.xq = xq; q.xs = xs; q.xbf = xbf; q.xq_out = xq_out; q.xs_out = xs_out;
  q.codes = ent; q.meta = nullptr; q.gamma = gamma; q.y = y; q.acc_out = acc;
  q.T = t; q.K = k; q.N = n_out; q.cstride = (int)entropy_row_bytes(k, n, m); q.mstride = 0;
  q.tiles_per_cta = per_cta;
  return t <= 8 ? dispatch_decode_ent<8, ACC, XBF>(q, n, m, grid, smem, cs)
                : dispatch_decode_ent<16, ACC, XBF>(q, n, m, grid, smem, cs);
}

template <bool ACC>
sbn_status run_bitlinear_entropy(const int8_t* xq, const float* xs, int32_t t, int32_t k, int32_t n_out,
                                 int32_t n, int32_t m, const uint8_t* ent, const float* gamma, uint16_t* y,
                                 int32_t* acc, void* stream) {
  sbn_status st = ent_decode_args(t, k, n_out, n, m);
  if (st != SBN_OK) return st;
  if (!aligned16(xq) || !aligned16(ent)) return SBN_ERR_ALIGN;
  int dev = 0, sms = 0;
  if ((st = check_device(&dev, &sms)) != SBN_OK) return st;
  int grid = 0, per_cta = 0;
  size_t smem = 0;
  if (!ent_decode_fits(t, k, n_out, n, m, sms, false, &grid, &per_cta, &smem)) return SBN_ERR_SHAPE;
  return launch_bitlinear_entropy<ACC, false>(xq, xs, nullptr, nullptr, nullptr, t, k, n_out, n, m, ent, gamma, y,
                                       acc, grid, per_cta, smem, reinterpret_cast<cudaStream_t>(stream));
}

// Workspace of sbn_bitlinear_entropy_x when it runs as two steps (Xq and s).
size_t bitlinear_entropy_x_ws_bytes(int32_t t, int32_t k) {
  return round_up16((size_t)t * k) + round_up16((size_t)t * 4);
}

// Backward dX over the packed weights, per pattern.
template <int MM, int CB, bool DENSE>
sbn_status launch_bwd_dx(const uint16_t* dy, int t, int k, int n_out, const uint8_t* codes, const uint8_t* meta,
                         int cstride, int mstride, const float* gamma, uint16_t* dx, cudaStream_t st) {
  const dim3 grid(k / kBwTile, (t + kBwTile - 1) / kBwTile);
  bwd_dx_kernel<MM, CB, DENSE><<<grid, kBwThreads, 0, st>>>(dy, t, k, n_out, codes, meta, cstride, mstride,
                                                           gamma, dx);
  return launch_status();
}

// dX on the tensor cores: dY [T, N_out] by TMA (N_out a multiple of 8, so
// its rows start on 16-byte boundaries), C expanded by the producer warps.
template <int MM, int CB, bool DENSE>
sbn_status launch_bwd_dx_tc(const uint16_t* dy, int t, int k, int n_out, const uint8_t* codes,
                            const uint8_t* meta, int cstride, int mstride, const float* gamma, uint16_t* dx,
                            int sms, cudaStream_t st) {
  static bool attr_set[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return SBN_ERR_CUDA;
  }
  auto kern = bwd_dx_tc_kernel<MM, CB, DENSE>;
  if (!attr_set[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kBxSmemBytes) !=
        cudaSuccess) {
      cudaGetLastError();
      return SBN_ERR_CUDA;
    }
    attr_set[dev] = true;
  }
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return SBN_ERR_CUDA;
  CUtensorMap tm;
  cuuint64_t gdim[2] = {(cuuint64_t)n_out, (cuuint64_t)t};
  cuuint64_t gstride[1] = {(cuuint64_t)n_out * 2};
  cuuint32_t box[2] = {(cuuint32_t)kBxBK, (cuuint32_t)kBxBM};
  cuuint32_t estride[2] = {1, 1};
  if (enc(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(dy), gdim, gstride, box, estride,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return SBN_ERR_CUDA;
  BxParams p;
  p.codes = codes; p.meta = meta; p.gamma = gamma; p.dx = dx;
  p.T = t; p.K = k; p.N = n_out; p.cstride = cstride; p.mstride = mstride;
  const int tiles = ((t + kBxBM - 1) / kBxBM) * ((k + kBxBN - 1) / kBxBN);
  kern<<<std::min(tiles, sms), kTcThreads, kBxSmemBytes, st>>>(tm, p);
  return launch_status();
}

sbn_status dispatch_bwd_dx(const uint16_t* dy, int t, int k, int n_out, int n, int m, const uint8_t* codes,
                           const uint8_t* meta, const float* gamma, uint16_t* dx, int sms, cudaStream_t st) {
  const int cs = (int)sbn_codes_row_bytes(k, n, m), ms = (int)sbn_meta_row_bytes(k, n, m);
  if ((n_out % 8) == 0) {
    if (n == m) return launch_bwd_dx_tc<8, 4, true>(dy, t, k, n_out, codes, meta, cs, ms, gamma, dx, sms, st);
    switch (m * 8 + 4 * n / m) {
      case 4 * 8 + 1: return launch_bwd_dx_tc<4, 1, false>(dy, t, k, n_out, codes, meta, cs, ms, gamma, dx, sms, st);
      case 4 * 8 + 2: return launch_bwd_dx_tc<4, 2, false>(dy, t, k, n_out, codes, meta, cs, ms, gamma, dx, sms, st);
      case 4 * 8 + 3: return launch_bwd_dx_tc<4, 3, false>(dy, t, k, n_out, codes, meta, cs, ms, gamma, dx, sms, st);
      case 8 * 8 + 1: return launch_bwd_dx_tc<8, 1, false>(dy, t, k, n_out, codes, meta, cs, ms, gamma, dx, sms, st);
      case 8 * 8 + 2: return launch_bwd_dx_tc<8, 2, false>(dy, t, k, n_out, codes, meta, cs, ms, gamma, dx, sms, st);
      case 8 * 8 + 3: return launch_bwd_dx_tc<8, 3, false>(dy, t, k, n_out, codes, meta, cs, ms, gamma, dx, sms, st);
      case 16 * 8 + 1: return launch_bwd_dx_tc<16, 1, false>(dy, t, k, n_out, codes, meta, cs, ms, gamma, dx, sms, st);
      case 16 * 8 + 2: return launch_bwd_dx_tc<16, 2, false>(dy, t, k, n_out, codes, meta, cs, ms, gamma, dx, sms, st);
      case 16 * 8 + 3: return launch_bwd_dx_tc<16, 3, false>(dy, t, k, n_out, codes, meta, cs, ms, gamma, dx, sms, st);
    }
    return SBN_ERR_PATTERN;
  }
  // N_out not a multiple of 8: the CUDA-core kernel
  if (n == m) return launch_bwd_dx<8, 4, true>(dy, t, k, n_out, codes, meta, cs, ms, gamma, dx, st);
  switch (m * 8 + 4 * n / m) {
    case 4 * 8 + 1: return launch_bwd_dx<4, 1, false>(dy, t, k, n_out, codes, meta, cs, ms, gamma, dx, st);
    case 4 * 8 + 2: return launch_bwd_dx<4, 2, false>(dy, t, k, n_out, codes, meta, cs, ms, gamma, dx, st);
    case 4 * 8 + 3: return launch_bwd_dx<4, 3, false>(dy, t, k, n_out, codes, meta, cs, ms, gamma, dx, st);
    case 8 * 8 + 1: return launch_bwd_dx<8, 1, false>(dy, t, k, n_out, codes, meta, cs, ms, gamma, dx, st);
    case 8 * 8 + 2: return launch_bwd_dx<8, 2, false>(dy, t, k, n_out, codes, meta, cs, ms, gamma, dx, st);
    case 8 * 8 + 3: return launch_bwd_dx<8, 3, false>(dy, t, k, n_out, codes, meta, cs, ms, gamma, dx, st);
    case 16 * 8 + 1: return launch_bwd_dx<16, 1, false>(dy, t, k, n_out, codes, meta, cs, ms, gamma, dx, st);
    case 16 * 8 + 2: return launch_bwd_dx<16, 2, false>(dy, t, k, n_out, codes, meta, cs, ms, gamma, dx, st);
    case 16 * 8 + 3: return launch_bwd_dx<16, 3, false>(dy, t, k, n_out, codes, meta, cs, ms, gamma, dx, st);
  }
  return SBN_ERR_PATTERN;
}

// Grid of the shard kernels: at most two waves of 512-thread CTAs.
int shard_grid(long long work_items, int sms) {
  const long long want = (work_items + kQbThreads - 1) / kQbThreads;
  return (int)std::max(1LL, std::min(want, (long long)sms * 4));
}

template <int M>
sbn_status launch_qw_from_bins(const uint16_t* w, int n_out, int k, int n, const unsigned long long* bins,
                               long long n_elems, uint8_t* codes, uint8_t* meta, float* gamma, int sms,
                               cudaStream_t st) {
  const int cstride = (int)sbn_codes_row_bytes(k, n, M);
  const int mstride = (int)sbn_meta_row_bytes(k, n, M);
  qw_from_bins_kernel<M><<<shard_grid((long long)n_out * (k / 16), sms), kQbThreads, 0, st>>>(
      w, n_out, k, n, bins, n_elems, codes, cstride, meta, mstride, gamma);
  return launch_status();
}

// Resident blocks per SM of the entropy packer (its grid fills the GPU once).
int ent_pack_blocks_per_sm(int dev, int m) {
  static int cached[kMaxDevices][3] = {};   // m = 4, 8, 16 (benign race: same value)
  const int mi = m == 4 ? 0 : (m == 8 ? 1 : 2);
  if (cached[dev][mi] == 0) {
    int b = 0;
    cudaError_t e = m == 4 ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, entropy_pack_kernel<4>, kEpThreads, 0)
                  : m == 8 ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, entropy_pack_kernel<8>, kEpThreads, 0)
                           : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, entropy_pack_kernel<16>, kEpThreads, 0);
    if (e != cudaSuccess) cudaGetLastError();
    cached[dev][mi] = std::max(1, b);
  }
  return cached[dev][mi];
}

// Fixed scratch of sbn_quantize_weights_noalloc (see include/sbn.h).
constexpr size_t kNoAllocScratchBytes = SBN_NOALLOC_SCRATCH_BYTES;
static_assert(kQwWorkspaceBytes <= kNoAllocScratchBytes, "workspace exceeds the fixed scratch");
void* g_noalloc_ptr[kMaxDevices];  // device address of g_noalloc_scratch, per device

}  // namespace

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

}  // namespace sbn

using namespace sbn;

extern "C" {

const char* sbn_status_string(sbn_status s) {
  switch (s) {
    case SBN_OK: return "SBN_OK";
    case SBN_ERR_NULL: return "SBN_ERR_NULL: a required pointer is NULL";
    case SBN_ERR_SHAPE: return "SBN_ERR_SHAPE: a size is out of the supported range";
    case SBN_ERR_PATTERN: return "SBN_ERR_PATTERN: unsupported n:m pattern";
    case SBN_ERR_ALIGN: return "SBN_ERR_ALIGN: a pointer is not 16-byte aligned";
    case SBN_ERR_WORKSPACE: return "SBN_ERR_WORKSPACE: workspace too small";
    case SBN_ERR_CUDA: return "SBN_ERR_CUDA: a CUDA call or launch failed";
    case SBN_ERR_TIMEOUT: return "SBN_ERR_TIMEOUT: a bounded device wait gave up";
    case SBN_ERR_DEVICE: return "SBN_ERR_DEVICE: the current device is not sm_100";
  }
  return "SBN_ERR_UNKNOWN";
}

int sbn_version(void) { return 100; }

size_t sbn_codes_row_bytes(int32_t k, int32_t n, int32_t m) {
  if (!pattern_ok(n, m) || k < 1 || (k % m) != 0) return 0;
  const size_t kept = (size_t)k / (size_t)m * (size_t)n;
  return round_up16((kept + 3) / 4);
}

size_t sbn_codes_bytes(int32_t n_out, int32_t k, int32_t n, int32_t m) {
  if (n_out < 1) return 0;
  return (size_t)n_out * sbn_codes_row_bytes(k, n, m);
}

size_t sbn_meta_row_bytes(int32_t k, int32_t n, int32_t m) {
  if (!pattern_ok(n, m) || k < 1 || (k % m) != 0 || n == m) return 0;
  return round_up16(((size_t)k + 7) / 8);
}

size_t sbn_meta_bytes(int32_t n_out, int32_t k, int32_t n, int32_t m) {
  if (n_out < 1) return 0;
  return (size_t)n_out * sbn_meta_row_bytes(k, n, m);
}

size_t sbn_quantize_weights_workspace_bytes(int32_t n_out, int32_t k) {
  (void)n_out;
  (void)k;
  return kQwWorkspaceBytes;
}

sbn_status sbn_quantize_weights(const void* w_bf16, int32_t n_out, int32_t k, int32_t n, int32_t m,
                                uint8_t* codes, uint8_t* meta, float* gamma, void* workspace,
                                size_t workspace_bytes, void* stream) {
  if (!w_bf16 || !codes || !gamma || !workspace || (n != m && !meta)) return SBN_ERR_NULL;
  sbn_status st = validate_weights_shape(n_out, k, n, m);
  if (st != SBN_OK) return st;
  if (!aligned16(w_bf16) || !aligned16(codes) || (meta && !aligned16(meta)) || !aligned16(workspace) ||
      (reinterpret_cast<uintptr_t>(gamma) & 3u))
    return SBN_ERR_ALIGN;
  if (workspace_bytes < kQwWorkspaceBytes) return SBN_ERR_WORKSPACE;
  int dev = 0, sms = 0;
  if ((st = check_device(&dev, &sms)) != SBN_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

  return launch_quantize_weights(reinterpret_cast<const uint16_t*>(w_bf16), n_out, k, n, m, codes,
                                 meta, gamma, reinterpret_cast<unsigned char*>(workspace), sms, s);
}

sbn_status sbn_quantize_acts(const void* x_bf16, int32_t t, int32_t k, int8_t* xq, float* x_scale,
                             void* stream) {
  if (!x_bf16 || !xq || !x_scale) return SBN_ERR_NULL;
  if (t < 1 || k < 16 || (k % 16) != 0 || !prod_lt_2_31(t, k)) return SBN_ERR_SHAPE;
  if (!aligned16(x_bf16) || !aligned16(xq) || (reinterpret_cast<uintptr_t>(x_scale) & 3u))
    return SBN_ERR_ALIGN;
  int dev = 0, sms = 0;
  sbn_status st = check_device(&dev, &sms);
  if (st != SBN_OK) return st;
  return launch_quantize_acts(x_bf16, t, k, xq, x_scale, sms, reinterpret_cast<cudaStream_t>(stream));
}

sbn_status sbn_mask_flips(const uint8_t* meta_a, const uint8_t* meta_b, int32_t n_out, int32_t k,
                          int32_t n, int32_t m, unsigned long long* flips, void* stream) {
  if (!meta_a || !meta_b || !flips) return SBN_ERR_NULL;
  if (!pattern_ok(n, m) || n == m) return SBN_ERR_PATTERN;
  if (n_out < 1 || k < 128 || (k % 128) != 0 || !prod_lt_2_31(n_out, k)) return SBN_ERR_SHAPE;
  if (!aligned16(meta_a) || !aligned16(meta_b) || (reinterpret_cast<uintptr_t>(flips) & 7u))
    return SBN_ERR_ALIGN;
  int dev = 0, sms = 0;
  sbn_status st = check_device(&dev, &sms);
  if (st != SBN_OK) return st;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(flips, 0, sizeof(unsigned long long), cs) != cudaSuccess) {
    cudaGetLastError();
    return SBN_ERR_CUDA;
  }
  // rows are padded with zero bytes in both masks, so the padding never counts
  const long long n16 = (long long)n_out * (long long)sbn_meta_row_bytes(k, n, m) / 16;
  const long long want = (n16 + kFlipThreads - 1) / kFlipThreads;
  const int grid = (int)std::max(1LL, std::min(want, (long long)sms * 8));
  flip_count_kernel<<<grid, kFlipThreads, 0, cs>>>(reinterpret_cast<const uint4*>(meta_a),
                                                   reinterpret_cast<const uint4*>(meta_b), n16, flips);
  return launch_status();
}

size_t sbn_entropy_row_bytes(int32_t k, int32_t n, int32_t m) {
  if (!pattern_ok(n, m) || k < 1 || (k % m) != 0) return 0;
  return entropy_row_bytes(k, n, m);
}

size_t sbn_entropy_bytes(int32_t n_out, int32_t k, int32_t n, int32_t m) {
  if (n_out < 1) return 0;
  return (size_t)n_out * sbn_entropy_row_bytes(k, n, m);
}

sbn_status sbn_pack_entropy(const uint8_t* codes, const uint8_t* meta, int32_t n_out, int32_t k,
                            int32_t n, int32_t m, uint8_t* ent, void* stream) {
  if (!codes || !ent || (n != m && !meta)) return SBN_ERR_NULL;
  sbn_status st = validate_weights_shape(n_out, k, n, m);
  if (st != SBN_OK) return st;
  if (!aligned16(codes) || !aligned16(ent) || (meta && !aligned16(meta))) return SBN_ERR_ALIGN;
  int dev = 0, sms = 0;
  if ((st = check_device(&dev, &sms)) != SBN_OK) return st;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  const int cws = (int)(sbn_codes_row_bytes(k, n, m) / 4);
  const int mws = (int)(sbn_meta_row_bytes(k, n, m) / 4);
  const int ews = (int)(sbn_entropy_row_bytes(k, n, m) / 4);
  EntPackParams prm;
  fill_ent_pack_params(prm, n, m);
  const long long segs = (k / m + 31) / 32;   // 32-group segments per row
  const long long items = (long long)n_out * ((segs + kEpUnroll - 1) / kEpUnroll);
  const int grid = (int)std::max(1LL, std::min((items + kEpWarps - 1) / kEpWarps,
                                               (long long)sms * ent_pack_blocks_per_sm(dev, m)));
  const uint32_t* c32 = reinterpret_cast<const uint32_t*>(codes);
  const uint32_t* m32 = reinterpret_cast<const uint32_t*>(meta);
  uint32_t* e32 = reinterpret_cast<uint32_t*>(ent);
  switch (m) {
    case 4: entropy_pack_kernel<4><<<grid, kEpThreads, 0, cs>>>(c32, m32, n_out, k, n, cws, mws, e32, ews, prm); break;
    case 8: entropy_pack_kernel<8><<<grid, kEpThreads, 0, cs>>>(c32, m32, n_out, k, n, cws, mws, e32, ews, prm); break;
    default: entropy_pack_kernel<16><<<grid, kEpThreads, 0, cs>>>(c32, m32, n_out, k, n, cws, mws, e32, ews, prm); break;
  }
  return launch_status();
}

sbn_status sbn_bitlinear_entropy(const int8_t* xq, const float* x_scale, int32_t t, int32_t k,
                                 int32_t n_out, int32_t n, int32_t m, const uint8_t* ent,
                                 const float* gamma, void* y_bf16, void* stream) {
  if (!xq || !x_scale || !ent || !gamma || !y_bf16) return SBN_ERR_NULL;
  if (!aligned16(y_bf16)) return SBN_ERR_ALIGN;
  return run_bitlinear_entropy<false>(xq, x_scale, t, k, n_out, n, m, ent, gamma,
                                      reinterpret_cast<uint16_t*>(y_bf16), nullptr, stream);
}

sbn_status sbn_bitlinear_entropy_acc32(const int8_t* xq, int32_t t, int32_t k, int32_t n_out, int32_t n,
                                       int32_t m, const uint8_t* ent, int32_t* acc, void* stream) {
  if (!xq || !ent || !acc) return SBN_ERR_NULL;
  if (!aligned16(acc)) return SBN_ERR_ALIGN;
  return run_bitlinear_entropy<true>(xq, nullptr, t, k, n_out, n, m, ent, nullptr, nullptr, acc, stream);
}

sbn_status sbn_bitlinear_grad_x(const void* dy_bf16, int32_t t, int32_t k, int32_t n_out, int32_t n, int32_t m,
                                const uint8_t* codes, const uint8_t* meta, const float* gamma, void* dx_bf16,
                                void* stream) {
  if (!dy_bf16 || !codes || !gamma || !dx_bf16 || (n != m && !meta)) return SBN_ERR_NULL;
  if (!pattern_ok(n, m)) return SBN_ERR_PATTERN;
  if (t < 1 || n_out < 1 || k < 128 || (k % 128) != 0) return SBN_ERR_SHAPE;
  if (!prod_lt_2_31(t, k) || !prod_lt_2_31(n_out, k) || !prod_lt_2_31(t, n_out)) return SBN_ERR_SHAPE;
  if ((t + kBwTile - 1) / kBwTile > 65535) return SBN_ERR_SHAPE;   // grid y
  if (!aligned16(dy_bf16) || !aligned16(codes) || (meta && !aligned16(meta)) || !aligned16(dx_bf16) ||
      (reinterpret_cast<uintptr_t>(gamma) & 3u))
    return SBN_ERR_ALIGN;
  int dev = 0, sms = 0;
  sbn_status st = check_device(&dev, &sms);
  if (st != SBN_OK) return st;
  return dispatch_bwd_dx(reinterpret_cast<const uint16_t*>(dy_bf16), t, k, n_out, n, m, codes, meta, gamma,
                         reinterpret_cast<uint16_t*>(dx_bf16), sms, reinterpret_cast<cudaStream_t>(stream));
}

sbn_status sbn_bitlinear_grad_w(const void* dy_bf16, const int8_t* xq, const float* x_scale, int32_t t,
                                int32_t k, int32_t n_out, void* dw_bf16, void* stream) {
  if (!dy_bf16 || !xq || !x_scale || !dw_bf16) return SBN_ERR_NULL;
  if (t < 1 || n_out < 1 || k < 128 || (k % 128) != 0) return SBN_ERR_SHAPE;
  if (!prod_lt_2_31(t, k) || !prod_lt_2_31(n_out, k) || !prod_lt_2_31(t, n_out)) return SBN_ERR_SHAPE;
  if ((n_out + kBwTile - 1) / kBwTile > 65535) return SBN_ERR_SHAPE;   // grid y
  if (!aligned16(dy_bf16) || !aligned16(xq) || !aligned16(dw_bf16) || (reinterpret_cast<uintptr_t>(x_scale) & 3u))
    return SBN_ERR_ALIGN;
  int dev = 0, sms = 0;
  sbn_status st = check_device(&dev, &sms);
  if (st != SBN_OK) return st;
  if ((n_out % 8) == 0 && t >= 32) {
    // tensor cores: the scaled dY split into two bf16 parts (2^-18 relative),
    // which needs at least 32 tokens to stay within the fp32 kernel's bound
    static bool attr_set[kMaxDevices] = {};
    if (!attr_set[dev]) {
      if (cudaFuncSetAttribute(bwd_dw_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kBwSmemBytes) !=
          cudaSuccess) {
        cudaGetLastError();
        return SBN_ERR_CUDA;
      }
      attr_set[dev] = true;
    }
    BwParams p;
    p.dy = reinterpret_cast<const uint16_t*>(dy_bf16); p.xq = xq; p.xs = x_scale;
    p.dw = reinterpret_cast<uint16_t*>(dw_bf16); p.T = t; p.K = k; p.N = n_out;
    const int tiles = ((n_out + kBwBM - 1) / kBwBM) * ((k + kBwBN - 1) / kBwBN);
    bwd_dw_tc_kernel<<<std::min(tiles, sms), kTcThreads, kBwSmemBytes, reinterpret_cast<cudaStream_t>(stream)>>>(p);
    return launch_status();
  }
  const dim3 grid(k / kBwTile, (n_out + kBwTile - 1) / kBwTile);
  bwd_dw_kernel<<<grid, kBwThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const uint16_t*>(dy_bf16), xq, x_scale, t, k, n_out, reinterpret_cast<uint16_t*>(dw_bf16));
  return launch_status();
}

size_t sbn_bitlinear_entropy_x_workspace_bytes(int32_t t, int32_t k) {
  if (t < 1 || k < 1) return 0;
  return bitlinear_entropy_x_ws_bytes(t, k);
}

sbn_status sbn_bitlinear_entropy_x(const void* x_bf16, int32_t t, int32_t k, int32_t n_out, int32_t n,
                                   int32_t m, const uint8_t* ent, const float* gamma, void* y_bf16,
                                   int8_t* xq, float* x_scale, void* workspace, size_t ws_bytes,
                                   void* stream) {
  if (!x_bf16 || !ent || !gamma || !y_bf16) return SBN_ERR_NULL;
  sbn_status st = ent_decode_args(t, k, n_out, n, m);
  if (st != SBN_OK) return st;
  if (!prod_lt_2_31(t, k) || !prod_lt_2_31(t, n_out)) return SBN_ERR_SHAPE;
  if (!aligned16(x_bf16) || !aligned16(ent) || !aligned16(y_bf16) || (xq && !aligned16(xq)) ||
      (reinterpret_cast<uintptr_t>(x_scale) & 3u) || (workspace && !aligned16(workspace)))
    return SBN_ERR_ALIGN;
  int dev = 0, sms = 0;
  if ((st = check_device(&dev, &sms)) != SBN_OK) return st;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  uint16_t* y = reinterpret_cast<uint16_t*>(y_bf16);
  int grid = 0, per_cta = 0;
  size_t smem = 0;
  if (ent_decode_fits(t, k, n_out, n, m, sms, true, &grid, &per_cta, &smem))
    return launch_bitlinear_entropy<false, true>(nullptr, nullptr, reinterpret_cast<const uint16_t*>(x_bf16),
                                                 xq, x_scale, t, k, n_out, n, m, ent, gamma, y, nullptr,
                                                 grid, per_cta, smem, cs);
  // two steps: quantize_acts into the given buffers or the workspace, then
  // the contraction over int8 activations
  if (!ent_decode_fits(t, k, n_out, n, m, sms, false, &grid, &per_cta, &smem)) return SBN_ERR_SHAPE;
  if ((!xq || !x_scale) && (!workspace || ws_bytes < bitlinear_entropy_x_ws_bytes(t, k)))
    return SBN_ERR_WORKSPACE;
  uint8_t* w8 = reinterpret_cast<uint8_t*>(workspace);
  int8_t* q8 = xq ? xq : reinterpret_cast<int8_t*>(w8);
  float* sc = x_scale ? x_scale : reinterpret_cast<float*>(w8 + round_up16((size_t)t * k));
  if ((st = launch_quantize_acts(x_bf16, t, k, q8, sc, sms, cs)) != SBN_OK) return st;
  return launch_bitlinear_entropy<false, false>(q8, sc, nullptr, nullptr, nullptr, t, k, n_out, n, m, ent,
                                                gamma, y, nullptr, grid, per_cta, smem, cs);
}

size_t sbn_bitlinear_x_workspace_bytes(int32_t t, int32_t k, int32_t n_out) {
  if (t < 1 || k < 1 || n_out < 1) return 0;
  return bitlinear_x_ws_bytes(t, k, n_out);
}

sbn_status sbn_bitlinear_x(const void* x_bf16, int32_t t, int32_t k, int32_t n_out, int32_t n,
                           int32_t m, const uint8_t* codes, const uint8_t* meta, const float* gamma,
                           void* y_bf16, int8_t* xq, float* x_scale, void* workspace,
                           size_t ws_bytes, void* stream) {
  if (!x_bf16 || !gamma || !y_bf16 || !codes || (n != m && !meta)) return SBN_ERR_NULL;
  if (!pattern_ok(n, m)) return SBN_ERR_PATTERN;
  if (t < 1 || n_out < 1 || k < 128 || (k % 128) != 0) return SBN_ERR_SHAPE;
  if (!prod_lt_2_31(t, k) || !prod_lt_2_31(n_out, k) || !prod_lt_2_31(t, n_out)) return SBN_ERR_SHAPE;
  if (!aligned16(x_bf16) || !aligned16(codes) || (meta && !aligned16(meta)) || !aligned16(y_bf16) ||
      (xq && !aligned16(xq)) || (reinterpret_cast<uintptr_t>(x_scale) & 3u) ||
      (workspace && !aligned16(workspace)))
    return SBN_ERR_ALIGN;
  int dev = 0, sms = 0;
  sbn_status st = check_device(&dev, &sms);
  if (st != SBN_OK) return st;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  int grid = 0, per_cta = 0;
  size_t smem = 0;
  if (gemv_fits(t, k, n_out, n, m, sms, true, &grid, &per_cta, &smem))
    return run_gemv<false, true>(nullptr, nullptr, reinterpret_cast<const uint16_t*>(x_bf16), xq, x_scale, t, k,
                                 n_out, n, m, codes, meta, gamma, reinterpret_cast<uint16_t*>(y_bf16), nullptr,
                                 grid, per_cta, smem, cs);
  if (fused_decode_fits(t, k, n_out, n, m, sms, &grid, &per_cta, &smem)) {
    DresParams q;
    q.xq = nullptr; q.xs = nullptr; q.xbf = reinterpret_cast<const uint16_t*>(x_bf16);
    q.xq_out = xq; q.xs_out = x_scale;
    q.codes = codes; q.meta = meta; q.gamma = gamma; q.y = reinterpret_cast<uint16_t*>(y_bf16);
    q.acc_out = nullptr;
    q.T = t; q.K = k; q.N = n_out;
    q.cstride = (int)sbn_codes_row_bytes(k, n, m); q.mstride = (int)sbn_meta_row_bytes(k, n, m);
    q.tiles_per_cta = per_cta;
    return t <= 8 ? dispatch_decode_res<8, false, true>(q, n, m, grid, smem, cs)
                  : dispatch_decode_res<16, false, true>(q, n, m, grid, smem, cs);
  }
  // two steps: quantize_acts into the given buffers or the workspace, then
  // the contraction (which expands the weights into the rest of it)
  if (!workspace || ws_bytes < bitlinear_x_ws_bytes(t, k, n_out)) return SBN_ERR_WORKSPACE;
  uint8_t* w8 = reinterpret_cast<uint8_t*>(workspace);
  int8_t* q8 = xq ? xq : reinterpret_cast<int8_t*>(w8);
  float* sc = x_scale ? x_scale : reinterpret_cast<float*>(w8 + round_up16((size_t)t * k));
  void* rest = w8 + round_up16((size_t)t * k) + round_up16((size_t)t * 4);
  if ((st = launch_quantize_acts(x_bf16, t, k, q8, sc, sms, cs)) != SBN_OK) return st;
  return run_bitlinear<false>(q8, sc, t, k, n_out, n, m, codes, meta, gamma,
                              reinterpret_cast<uint16_t*>(y_bf16), nullptr,
                              bitlinear_ws_bytes(t, k, n_out) ? rest : nullptr, sms, cs);
}

size_t sbn_bitlinear_workspace_bytes(int32_t t, int32_t k, int32_t n_out) {
  if (t < 1 || k < 1 || n_out < 1) return 0;
  return bitlinear_ws_bytes(t, k, n_out);
}

sbn_status sbn_bitlinear(const int8_t* xq, const float* x_scale, int32_t t, int32_t k, int32_t n_out,
                         int32_t n, int32_t m, const uint8_t* codes, const uint8_t* meta,
                         const float* gamma, void* y_bf16, void* workspace, size_t ws_bytes,
                         void* stream) {
  if (!x_scale || !gamma || !y_bf16) return SBN_ERR_NULL;
  sbn_status st = validate_bitlinear(xq, t, k, n_out, n, m, codes, meta);
  if (st != SBN_OK) return st;
  if (!aligned16(y_bf16)) return SBN_ERR_ALIGN;
  if ((st = check_bitlinear_ws(t, k, n_out, workspace, ws_bytes)) != SBN_OK) return st;
  int dev = 0, sms = 0;
  if ((st = check_device(&dev, &sms)) != SBN_OK) return st;
  return run_bitlinear<false>(xq, x_scale, t, k, n_out, n, m, codes, meta, gamma,
                              reinterpret_cast<uint16_t*>(y_bf16), nullptr, workspace, sms,
                              reinterpret_cast<cudaStream_t>(stream));
}

sbn_status sbn_bitlinear_acc32(const int8_t* xq, int32_t t, int32_t k, int32_t n_out, int32_t n,
                               int32_t m, const uint8_t* codes, const uint8_t* meta, int32_t* acc,
                               void* workspace, size_t ws_bytes, void* stream) {
  if (!acc) return SBN_ERR_NULL;
  sbn_status st = validate_bitlinear(xq, t, k, n_out, n, m, codes, meta);
  if (st != SBN_OK) return st;
  if (!aligned16(acc)) return SBN_ERR_ALIGN;
  if ((st = check_bitlinear_ws(t, k, n_out, workspace, ws_bytes)) != SBN_OK) return st;
  int dev = 0, sms = 0;
  if ((st = check_device(&dev, &sms)) != SBN_OK) return st;
  return run_bitlinear<true>(xq, nullptr, t, k, n_out, n, m, codes, meta, nullptr, nullptr, acc,
                             workspace, sms, reinterpret_cast<cudaStream_t>(stream));
}

// Allocation-free variant of sbn_quantize_weights. Its scratch is a fixed
// array in this file; the host side only ever uses the device address that
// cudaGetSymbolAddress returns for it (looked up once per device, with that
// device current). The bins are cleared on every call, on the caller's stream.
sbn_status sbn_quantize_weights_noalloc(const void* w_bf16, int32_t n_out, int32_t k, int32_t n,
                                        int32_t m, uint8_t* codes, uint8_t* meta, float* gamma,
                                        void* stream) {
  if (!w_bf16 || !codes || !gamma || (n != m && !meta)) return SBN_ERR_NULL;
  sbn_status st = validate_weights_shape(n_out, k, n, m);
  if (st != SBN_OK) return st;
  if (!aligned16(w_bf16) || !aligned16(codes) || (meta && !aligned16(meta)) ||
      (reinterpret_cast<uintptr_t>(gamma) & 3u))
    return SBN_ERR_ALIGN;
  if (sbn_quantize_weights_workspace_bytes(n_out, k) > kNoAllocScratchBytes) return SBN_ERR_WORKSPACE;
  int dev = 0, sms = 0;
  if ((st = check_device(&dev, &sms)) != SBN_OK) return st;
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return SBN_ERR_CUDA;
    }
    g_noalloc_ptr[dev] = p;
  }
  return launch_quantize_weights(reinterpret_cast<const uint16_t*>(w_bf16), n_out, k, n, m, codes,
                                 meta, gamma, reinterpret_cast<unsigned char*>(g_noalloc_ptr[dev]), sms,
                                 reinterpret_cast<cudaStream_t>(stream));
}

sbn_status sbn_gamma_bins(const void* w_bf16, int32_t n_out, int32_t k, unsigned long long* bins,
                          void* stream) {
  if (!w_bf16 || !bins) return SBN_ERR_NULL;
  if (n_out < 1 || k < 128 || (k % 128) != 0 || !prod_lt_2_31(n_out, k)) return SBN_ERR_SHAPE;
  if (!aligned16(w_bf16) || !aligned16(bins)) return SBN_ERR_ALIGN;
  int dev = 0, sms = 0;
  sbn_status st = check_device(&dev, &sms);
  if (st != SBN_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(bins, 0, SBN_GAMMA_BINS * sizeof(unsigned long long), s) != cudaSuccess) {
    cudaGetLastError();
    return SBN_ERR_CUDA;
  }
  const long long chunks = (long long)n_out * k / 8;
  gamma_bins_kernel<<<shard_grid(chunks, sms), kQbThreads, 0, s>>>(reinterpret_cast<const uint4*>(w_bf16), chunks,
                                                                  bins);
  return launch_status();
}

sbn_status sbn_quantize_weights_from_bins(const void* w_bf16, int32_t n_out, int32_t k, int32_t n, int32_t m,
                                          const unsigned long long* bins, int64_t total_elems, uint8_t* codes,
                                          uint8_t* meta, float* gamma, void* stream) {
  if (!w_bf16 || !bins || !codes || !gamma || (n != m && !meta)) return SBN_ERR_NULL;
  sbn_status st = validate_weights_shape(n_out, k, n, m);
  if (st != SBN_OK) return st;
  if (total_elems < (int64_t)n_out * k || total_elems > (1ll << 36)) return SBN_ERR_SHAPE;
  if (!aligned16(w_bf16) || !aligned16(bins) || !aligned16(codes) || (meta && !aligned16(meta)) ||
      (reinterpret_cast<uintptr_t>(gamma) & 3u))
    return SBN_ERR_ALIGN;
  int dev = 0, sms = 0;
  if ((st = check_device(&dev, &sms)) != SBN_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const uint16_t* w = reinterpret_cast<const uint16_t*>(w_bf16);
  switch (m) {
    case 4: return launch_qw_from_bins<4>(w, n_out, k, n, bins, total_elems, codes, meta, gamma, sms, s);
    case 8: return launch_qw_from_bins<8>(w, n_out, k, n, bins, total_elems, codes, meta, gamma, sms, s);
    default: return launch_qw_from_bins<16>(w, n_out, k, n, bins, total_elems, codes, meta, gamma, sms, s);
  }
}

sbn_status sbn_probe_i8_mma(int32_t iters, int32_t* ctas, void* stream) {
  if (!ctas) return SBN_ERR_NULL;
  if (iters < 1 || iters > (1 << 24)) return SBN_ERR_SHAPE;
  int dev = 0, sms = 0;
  sbn_status st = check_device(&dev, &sms);
  if (st != SBN_OK) return st;
  static bool attr_set[kMaxDevices] = {};
  if (!attr_set[dev]) {
    if (cudaFuncSetAttribute(i8_peak_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kPkSmemBytes) !=
        cudaSuccess) {
      cudaGetLastError();
      return SBN_ERR_CUDA;
    }
    attr_set[dev] = true;
  }
  i8_peak_kernel<<<sms, kPkThreads, kPkSmemBytes, reinterpret_cast<cudaStream_t>(stream)>>>(iters);
  *ctas = sms;
  return launch_status();
}

sbn_status sbn_probe_i8_sparse_mma(int32_t iters, int32_t* pairs, void* stream) {
  if (!pairs) return SBN_ERR_NULL;
  if (iters < 1 || iters > (1 << 24)) return SBN_ERR_SHAPE;
  int dev = 0, sms = 0;
  sbn_status st = check_device(&dev, &sms);
  if (st != SBN_OK) return st;
  static int cached[kMaxDevices];   // 0 unknown, else resident pairs + 1
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaFuncSetAttribute(i8_sparse_peak_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kPsSmemBytes) == cudaSuccess) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(2);
      cfg.blockDim = dim3(kPkThreads);
      cfg.dynamicSmemBytes = kPsSmemBytes;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      if (cudaOccupancyMaxActiveClusters(&n, i8_sparse_peak_kernel, &cfg) != cudaSuccess) n = 0;
    }
    cudaGetLastError();
    cached[dev] = n + 1;
  }
  const int np = std::min(cached[dev] - 1, sms / 2);
  if (np <= 0) return SBN_ERR_DEVICE;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * np);
  cfg.blockDim = dim3(kPkThreads);
  cfg.dynamicSmemBytes = kPsSmemBytes;
  cfg.stream = reinterpret_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, i8_sparse_peak_kernel, (int)iters) != cudaSuccess) {
    cudaGetLastError();
    return SBN_ERR_CUDA;
  }
  *pairs = np;
  return launch_status();
}

sbn_status sbn_selftest_wait_timeout(int32_t which, int64_t limit_ns, void* stream) {
  if (which != 0 && which != 1) return SBN_ERR_SHAPE;
  if (limit_ns < 1000 || limit_ns > 100000000) return SBN_ERR_SHAPE;
  int dev = 0, sms = 0;
  sbn_status st = check_device(&dev, &sms);
  if (st != SBN_OK) return st;
  wait_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(which, (unsigned long long)limit_ns);
  return launch_status();
}

int32_t sbn_set_programmatic_launch(int32_t enable) {
  return sbn::g_pdl.exchange(enable ? 1 : 0);
}

sbn_status sbn_get_device_error(void* stream) {
  int dev = 0, sms = 0;
  sbn_status st = check_device(&dev, &sms);
  if (st != SBN_OK) return st;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return SBN_ERR_CUDA;
  }
  unsigned int v = 0u;
  const unsigned int zero = 0u;
  if (cudaMemcpyFromSymbol(&v, g_dev_error, sizeof(v)) != cudaSuccess ||
      cudaMemcpyToSymbol(g_dev_error, &zero, sizeof(zero)) != cudaSuccess) {
    cudaGetLastError();
    return SBN_ERR_CUDA;
  }
  return v == kDevErrNone ? SBN_OK : SBN_ERR_TIMEOUT;
}

}  // extern "C"
