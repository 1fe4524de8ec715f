// attn_bwd.cu - backward attention kernels for sm_100a (being written).
#include <cuda_runtime.h>
#include "../../include/tiledattn.h"

extern "C" int attn_bwd(const void*, const void*, const void*, const void*, const float*, const void*, void*, void*,
                        void*, int, int, int, int, int, int, float, int, int, void*, size_t, void*) {
  return ATTN_ERR_UNSUPPORTED;
}
