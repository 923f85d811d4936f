// ABI plumbing shared by every entry point: status strings, version, per-thread last CUDA error.
#include "csa_common.cuh"

namespace csa {
static thread_local int g_last_cuda_error = 0;
void set_last_cuda_error(cudaError_t e) { g_last_cuda_error = (int)e; }
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
