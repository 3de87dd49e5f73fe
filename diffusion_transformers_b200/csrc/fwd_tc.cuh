// fwd_tc.cuh — tensor-core (tcgen05) engines. Placeholder until the kernels land.
#pragma once
#include <string>
#include "common.cuh"
#include "binattn.h"

namespace binattn {

inline bool tc_supported(int d) { return d % 8 == 0 && d <= 128; }
inline bool tc_built() { return false; }

inline int forward_tc(bool, const uint32_t*, const uint32_t*, const float*, const float*,
                      const uint16_t*, const uint16_t*, float, int, int, int, int, uint16_t*,
                      cudaStream_t, std::string* msg) {
  *msg = "tensor-core engines are not built yet";
  return BINATTN_ERR_UNSUPPORTED;
}
inline int scores_tc(const uint32_t*, const uint32_t*, int, int, int, int, int32_t*, cudaStream_t,
                     std::string* msg) {
  *msg = "tensor-core engines are not built yet";
  return BINATTN_ERR_UNSUPPORTED;
}
inline int forward_ref_bf16(const uint16_t*, const uint16_t*, const uint16_t*, const uint16_t*, float,
                            int, int, int, int, uint16_t*, cudaStream_t, std::string* msg) {
  *msg = "bf16 reference not built yet";
  return BINATTN_ERR_UNSUPPORTED;
}

}  // namespace binattn
