// Verify attention (placeholder until the tcgen05 kernel lands).
#include "vc_internal.h"

namespace vc {

size_t verify_workspace_bytes(int, int, int, int, int, int64_t, int64_t) { return 256; }

vc_status launch_verify(const void*, int, int, int, int, int, const void*, const void*, int64_t,
                        int64_t, int64_t, int64_t, float*, float*, float*, int, float, void*,
                        void*, size_t, cudaStream_t) {
  return fail(VC_ERR_UNSUPPORTED, "verify attention not built yet");
}

}  // namespace vc
