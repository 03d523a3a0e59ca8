// Backward pass (placeholder until the tcgen05 backward lands).
#include "../../include/ba.h"

extern "C" ba_status ba_bwd(const ba_problem*, const void*, const void*, const float*,
                            const void*, const void*, void*, void*, void*, void*, void*, void*,
                            ba_stream_t) {
  return BA_ERR_UNSUPPORTED;
}
