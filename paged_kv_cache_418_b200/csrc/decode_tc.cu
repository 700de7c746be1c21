// decode_tc.cu -- tcgen05 (5th-generation tensor core) path for grouped-query
// decode attention. Placeholder until the kernel lands: reports "not supported"
// so the planner keeps every shape on the CUDA-core path.
#include "pa_internal.h"

namespace pa {

bool tc_supported(int dtype, int Hq, int Hkv, int D, int bs) {
  (void)dtype; (void)Hq; (void)Hkv; (void)D; (void)bs;
  return false;
}

int launch_decode_tc(const DecodeArgs& a, int dtype, cudaStream_t stream) {
  (void)a; (void)dtype; (void)stream;
  return PA_ERR_UNSUPPORTED;
}

}  // namespace pa
