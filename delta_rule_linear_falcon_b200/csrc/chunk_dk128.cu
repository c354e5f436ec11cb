// chunk_dk128.cu -- chunk-parallel kernel instantiations for d_k = 128.
#include "chunk_kernel.cuh"

namespace falcon {
FALCON_CHUNK_DK_DISPATCH(128)
}  // namespace falcon
