// Entry points whose kernels are not in this build yet: they report
// LLA_ERR_UNSUPPORTED without touching the device.
#include "internal.h"

using namespace lla;

extern "C" {

size_t lla2d_decode_attn_workspace(int, int, int, int, int) { return 0; }

lla_status lla2d_decode_attn(const float*, const void*, const void*, lla_dtype, int, int, int,
                             int, int, int, int, const float*, const float*, const float*,
                             const float*, float, float*, float*, void*, size_t, void*) {
  return fail(LLA_ERR_UNSUPPORTED, "lla2d_decode_attn is not built yet");
}

}  // extern "C"
