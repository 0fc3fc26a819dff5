// Library-wide entry points of libmsa: status strings, CUDA error capture,
// the per-device status word.
#include <mutex>
#include <map>
#include <utility>

#include "msa_common.cuh"

namespace msa {

namespace {
thread_local int t_last_cuda_error = 0;

constexpr int kMaxDevices = 64;
std::mutex g_mu;
int* g_status_ptr[kMaxDevices] = {};
int g_sms[kMaxDevices] = {};
}  // namespace

// Status word of each device: first device-detected error since the last
// msa_device_status(..., clear=1).
__device__ int g_device_status = 0;

int note_cuda(cudaError_t e) {
  if (e == cudaSuccess) return MSA_OK;
  t_last_cuda_error = static_cast<int>(e);
  return MSA_ERR_CUDA;
}

static int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  return dev;
}

int* device_status_ptr() {
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_status_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    g_status_ptr[dev] = static_cast<int*>(p);
  }
  return g_status_ptr[dev];
}

int num_sms() {
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return 148;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_sms[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) !=
            cudaSuccess ||
        n <= 0) {
      cudaGetLastError();
      n = 148;
    }
    g_sms[dev] = n;
  }
  return g_sms[dev];
}

int ensure_smem_attr(const void* func, int bytes) {
  // The attribute is one value per (kernel, device): keep the largest value
  // set so far and only ever raise it.
  const int dev = current_device();
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, int> limit;
  std::lock_guard<std::mutex> lk(mu);
  const auto key = std::make_pair(func, dev);
  const auto it = limit.find(key);
  if (it != limit.end() && it->second >= bytes) return MSA_OK;
  const int rc = note_cuda(
      cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes));
  if (rc == MSA_OK) limit[key] = bytes;
  return rc;
}

}  // namespace msa

extern "C" {

const char* msa_status_string(int status) {
  switch (status) {
    case MSA_OK: return "ok";
    case MSA_ERR_INVALID_ARG: return "invalid argument";
    case MSA_ERR_UNSUPPORTED: return "unsupported shape or type";
    case MSA_ERR_CAPACITY: return "memory capacity exceeded";
    case MSA_ERR_CUDA: return "CUDA error";
    case MSA_ERR_TIMEOUT: return "device wait timed out";
    case MSA_ERR_WORKSPACE: return "workspace missing or too small";
    default: return "unknown status";
  }
}

int msa_last_cuda_error(void) { return msa::t_last_cuda_error; }

const char* msa_version(void) { return "libmsa 0.1.0 sm_100a"; }

int msa_device_status(int32_t* host_out, int clear, msa_stream_t stream) {
  if (!host_out) return MSA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int* dptr = msa::device_status_ptr();
  if (!dptr) return msa::note_cuda(cudaErrorInvalidDevice);
  int v = 0;
  int rc = msa::note_cuda(
      cudaMemcpyAsync(&v, dptr, sizeof(int), cudaMemcpyDeviceToHost, s));
  if (rc) return rc;
  if (clear) {
    rc = msa::note_cuda(cudaMemsetAsync(dptr, 0, sizeof(int), s));
    if (rc) return rc;
  }
  rc = msa::note_cuda(cudaStreamSynchronize(s));
  if (rc) return rc;
  *host_out = v;
  return MSA_OK;
}

}  // extern "C"
