// Library-wide entry points of the C ABI: version and status strings.
#include "tcq_device.cuh"

extern "C" int tcq_version(void) { return 100; }   // 0.1.0

extern "C" const char *tcq_status_string(tcq_status_t status) {
  switch (status) {
    case TCQ_OK: return "ok";
    case TCQ_ERR_INVALID_ARG: return "invalid argument (null pointer, size, alignment or enum)";
    case TCQ_ERR_UNSUPPORTED: return "unsupported trellis, layout or size";
    case TCQ_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case TCQ_ERR_CUDA: return "CUDA launch or runtime call failed";
  }
  return "unknown status";
}
