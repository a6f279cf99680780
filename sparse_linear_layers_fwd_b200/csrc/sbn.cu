// libsbn: C ABI of the Sparse-BitNet BitLinear forward (see include/sbn.h).
//
// Host side of the library: argument validation (before anything touches
// the GPU), device checks, and the launches on the caller's stream. Every
// step of the path runs in the kernels included below; there is no host or
// CPU fallback.

#include "sbn.h"

#include <algorithm>
#include <climits>
#include <cstdint>
#include <cstring>

#include "common.cuh"
#include "qa.cuh"
#include "qw.cuh"
#include "bl_simt.cuh"

namespace sbn {

__device__ unsigned int g_dev_error;

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

sbn_status validate_weights_shape(int32_t n_out, int32_t k, int32_t n, int32_t m) {
  if (!pattern_ok(n, m)) return SBN_ERR_PATTERN;
  if (n_out < 1 || k < 128 || (k % 128) != 0) return SBN_ERR_SHAPE;
  if (!prod_lt_2_31(n_out, k)) return SBN_ERR_SHAPE;
  return SBN_OK;
}

template <int M>
void launch_pack(const uint16_t* w, int n_out, int k, int n, const uint32_t* tau, uint8_t* codes,
                 int cstride, uint8_t* meta, int mstride, int sms, cudaStream_t st) {
  const int blocks = (int)std::min<long long>((n_out + 7) / 8, (long long)sms * 4);
  qw_pack_kernel<M><<<blocks, 256, 0, st>>>(w, n_out, k, n, tau, codes, cstride, meta, mstride);
}

template <bool ACC_OUT>
sbn_status run_bitlinear(const int8_t* xq, const float* xs, int32_t t, int32_t k, int32_t n_out,
                         int32_t n, int32_t m, const uint8_t* codes, const uint8_t* meta,
                         const float* gamma, uint16_t* y, int32_t* acc, cudaStream_t st) {
  const int cstride = (int)sbn_codes_row_bytes(k, n, m);
  const int mstride = (int)sbn_meta_row_bytes(k, n, m);
  dim3 grid((n_out + kSimtO - 1) / kSimtO, (t + kSimtT - 1) / kSimtT);
  switch (m) {
    case 4:
      bl_simt_kernel<4, ACC_OUT><<<grid, 256, 0, st>>>(xq, xs, t, k, n_out, n, codes, cstride, meta,
                                                       mstride, gamma, y, acc);
      break;
    case 8:
      bl_simt_kernel<8, ACC_OUT><<<grid, 256, 0, st>>>(xq, xs, t, k, n_out, n, codes, cstride, meta,
                                                       mstride, gamma, y, acc);
      break;
    default:
      bl_simt_kernel<16, ACC_OUT><<<grid, 256, 0, st>>>(xq, xs, t, k, n_out, n, codes, cstride,
                                                        meta, mstride, gamma, y, acc);
      break;
  }
  return launch_status();
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

  unsigned long long* bins = reinterpret_cast<unsigned long long*>(workspace);
  uint32_t* tau = reinterpret_cast<uint32_t*>(reinterpret_cast<char*>(workspace) + kQwTauOffset);
  if (cudaMemsetAsync(bins, 0, kQwBins * sizeof(unsigned long long), s) != cudaSuccess) {
    cudaGetLastError();
    return SBN_ERR_CUDA;
  }
  const long long n_elems = (long long)n_out * k;
  const long long nchunks = n_elems / 8;
  const int blocks = (int)std::max<long long>(1, std::min<long long>((nchunks + 255) / 256, (long long)sms * 8));
  qw_bins_kernel<<<blocks, 256, 0, s>>>(reinterpret_cast<const uint4*>(w_bf16), nchunks, bins);
  qw_finalize_kernel<<<1, 32, 0, s>>>(bins, n_elems, gamma, tau);
  const uint16_t* w = reinterpret_cast<const uint16_t*>(w_bf16);
  const int cstride = (int)sbn_codes_row_bytes(k, n, m);
  const int mstride = (int)sbn_meta_row_bytes(k, n, m);
  switch (m) {
    case 4: launch_pack<4>(w, n_out, k, n, tau, codes, cstride, meta, mstride, sms, s); break;
    case 8: launch_pack<8>(w, n_out, k, n, tau, codes, cstride, meta, mstride, sms, s); break;
    default: launch_pack<16>(w, n_out, k, n, tau, codes, cstride, meta, mstride, sms, s); break;
  }
  return launch_status();
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
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int kc = k / 8;
  const uint4* x = reinterpret_cast<const uint4*>(x_bf16);
  uint2* q = reinterpret_cast<uint2*>(xq);
  const int need = (kc + kQaThreads - 1) / kQaThreads;
  if (need <= 1) qa_kernel<1><<<t, kQaThreads, 0, s>>>(x, kc, q, x_scale);
  else if (need <= 2) qa_kernel<2><<<t, kQaThreads, 0, s>>>(x, kc, q, x_scale);
  else if (need <= 4) qa_kernel<4><<<t, kQaThreads, 0, s>>>(x, kc, q, x_scale);
  else if (need <= 8) qa_kernel<8><<<t, kQaThreads, 0, s>>>(x, kc, q, x_scale);
  else if (need <= 12) qa_kernel<12><<<t, kQaThreads, 0, s>>>(x, kc, q, x_scale);
  else if (need <= 16) qa_kernel<16><<<t, kQaThreads, 0, s>>>(x, kc, q, x_scale);
  else qa_kernel_long<<<t, kQaThreads, 0, s>>>(x, kc, q, x_scale);
  return launch_status();
}

sbn_status sbn_bitlinear(const int8_t* xq, const float* x_scale, int32_t t, int32_t k, int32_t n_out,
                         int32_t n, int32_t m, const uint8_t* codes, const uint8_t* meta,
                         const float* gamma, void* y_bf16, void* stream) {
  if (!x_scale || !gamma || !y_bf16) return SBN_ERR_NULL;
  sbn_status st = validate_bitlinear(xq, t, k, n_out, n, m, codes, meta);
  if (st != SBN_OK) return st;
  if (!aligned16(y_bf16)) return SBN_ERR_ALIGN;
  int dev = 0, sms = 0;
  if ((st = check_device(&dev, &sms)) != SBN_OK) return st;
  return run_bitlinear<false>(xq, x_scale, t, k, n_out, n, m, codes, meta, gamma,
                              reinterpret_cast<uint16_t*>(y_bf16), nullptr,
                              reinterpret_cast<cudaStream_t>(stream));
}

sbn_status sbn_bitlinear_acc32(const int8_t* xq, int32_t t, int32_t k, int32_t n_out, int32_t n,
                               int32_t m, const uint8_t* codes, const uint8_t* meta, int32_t* acc,
                               void* stream) {
  if (!acc) return SBN_ERR_NULL;
  sbn_status st = validate_bitlinear(xq, t, k, n_out, n, m, codes, meta);
  if (st != SBN_OK) return st;
  if (!aligned16(acc)) return SBN_ERR_ALIGN;
  int dev = 0, sms = 0;
  if ((st = check_device(&dev, &sms)) != SBN_OK) return st;
  return run_bitlinear<true>(xq, nullptr, t, k, n_out, n, m, codes, meta, nullptr, nullptr, acc,
                             reinterpret_cast<cudaStream_t>(stream));
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
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  char* scratch = reinterpret_cast<char*>(g_noalloc_ptr[dev]);
  unsigned long long* bins = reinterpret_cast<unsigned long long*>(scratch);
  uint32_t* tau = reinterpret_cast<uint32_t*>(scratch + kQwTauOffset);
  if (cudaMemsetAsync(bins, 0, kQwBins * sizeof(unsigned long long), s) != cudaSuccess) {
    cudaGetLastError();
    return SBN_ERR_CUDA;
  }
  const long long n_elems = (long long)n_out * k;
  const long long nchunks = n_elems / 8;
  const int blocks = (int)std::max<long long>(1, std::min<long long>((nchunks + 255) / 256, (long long)sms * 8));
  qw_bins_kernel<<<blocks, 256, 0, s>>>(reinterpret_cast<const uint4*>(w_bf16), nchunks, bins);
  qw_finalize_kernel<<<1, 32, 0, s>>>(bins, n_elems, gamma, tau);
  const uint16_t* w = reinterpret_cast<const uint16_t*>(w_bf16);
  const int cstride = (int)sbn_codes_row_bytes(k, n, m);
  const int mstride = (int)sbn_meta_row_bytes(k, n, m);
  switch (m) {
    case 4: launch_pack<4>(w, n_out, k, n, tau, codes, cstride, meta, mstride, sms, s); break;
    case 8: launch_pack<8>(w, n_out, k, n, tau, codes, cstride, meta, mstride, sms, s); break;
    default: launch_pack<16>(w, n_out, k, n, tau, codes, cstride, meta, mstride, sms, s); break;
  }
  return launch_status();
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
