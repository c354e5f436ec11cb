// chunk_dk64.cu -- chunk-parallel kernel instantiations for d_k = 64.
#include "chunk_kernel.cuh"

namespace falcon {
FALCON_CHUNK_DK_DISPATCH(64)
}  // namespace falcon
