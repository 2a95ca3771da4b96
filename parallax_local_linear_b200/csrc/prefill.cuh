// Parallax causal prefill (tcgen05 / TMEM / TMA) -- under construction.
#pragma once

#include "ptx.cuh"

namespace plx {

inline plx_status launch_prefill(const void*, const void*, const void*, const void*, void*,
                                 const plx_prefill_params*, cudaStream_t) {
  return PLX_ERR_UNSUPPORTED;
}

}  // namespace plx
