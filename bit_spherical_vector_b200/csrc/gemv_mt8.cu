// gemv_mt8.cu -- GEMV kernel instantiation for 8 token(s) per pass
// (one translation unit per batch width so the builds run in parallel).
#include "gemv_impl.cuh"

namespace svq {
template cudaError_t launch_gemv_mt<8>(const GemvKParams&, int, size_t, cudaStream_t);
}  // namespace svq
