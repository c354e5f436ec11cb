// chunk_dk32.cu -- chunk-parallel kernel instantiations for d_k = 32.
#include "chunk_kernel.cuh"

namespace falcon {
FALCON_CHUNK_DK_DISPATCH(32)
}  // namespace falcon
