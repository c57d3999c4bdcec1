// Host-side helpers shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>

#include "../../include/tl.h"

namespace tl {

// Records the CUDA error text for tl_last_cuda_error() and maps it to a status.
int check_cuda(cudaError_t e);

}  // namespace tl

#define TL_CUDA(call)                        \
  do {                                       \
    int _st = ::tl::check_cuda((call));      \
    if (_st != TL_OK) return _st;            \
  } while (0)

#define TL_TRY(call)                         \
  do {                                       \
    int _st = (call);                        \
    if (_st != TL_OK) return _st;            \
  } while (0)
