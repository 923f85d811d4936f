// ABI plumbing shared by every entry point: status strings, version, per-thread last CUDA error.
#include "csa_common.cuh"

namespace csa {
static thread_local int g_last_cuda_error = 0;
void set_last_cuda_error(cudaError_t e) { g_last_cuda_error = (int)e; }

// The device error word's readers, one per translation unit, added while the library loads.
static std::atomic<DeviceErrorReader>* error_readers(int* cap) {
  static std::atomic<DeviceErrorReader> readers[32];
  *cap = 32;
  return readers;
}

void register_device_error_reader(DeviceErrorReader f) {
  int cap = 0;
  std::atomic<DeviceErrorReader>* r = error_readers(&cap);
  for (int i = 0; i < cap; ++i) {
    DeviceErrorReader expected = nullptr;
    if (r[i].compare_exchange_strong(expected, f)) return;
  }
}

int device_error_reader_count() {
  int cap = 0, n = 0;
  std::atomic<DeviceErrorReader>* r = error_readers(&cap);
  while (n < cap && r[n].load() != nullptr) ++n;
  return n;
}
}  // namespace csa

extern "C" const char* csa_status_string(int s) {
  switch (s) {
    case CSA_OK: return "CSA_OK";
    case CSA_ERR_INVALID: return "CSA_ERR_INVALID";
    case CSA_ERR_UNSUPPORTED: return "CSA_ERR_UNSUPPORTED";
    case CSA_ERR_WORKSPACE: return "CSA_ERR_WORKSPACE";
    case CSA_ERR_CUDA: return "CSA_ERR_CUDA";
    case CSA_ERR_DEVICE: return "CSA_ERR_DEVICE";
    default: return "CSA_ERR_UNKNOWN";
  }
}

extern "C" int csa_version(void) { return 100; }

extern "C" int csa_last_cuda_error(void) { return csa::g_last_cuda_error; }

extern "C" csa_status csa_device_status(void* stream) {
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  uint32_t v = 0;
  int cap = 0;
  std::atomic<csa::DeviceErrorReader>* r = csa::error_readers(&cap);
  for (int i = 0; i < cap && e == cudaSuccess; ++i) {
    const csa::DeviceErrorReader f = r[i].load();
    if (f == nullptr) break;
    e = f(&v);
  }
  if (e != cudaSuccess) {
    csa::set_last_cuda_error(e);
    return CSA_ERR_CUDA;
  }
  return v ? CSA_ERR_DEVICE : CSA_OK;
}
