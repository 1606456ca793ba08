// gemv_mt2.cu -- GEMV kernel instantiation for 2 token(s) per pass
// (one translation unit per batch width so the builds run in parallel).
#include "gemv_impl.cuh"

namespace svq {
template cudaError_t launch_gemv_mt<2>(const GemvKParams&, int, size_t, cudaStream_t);
}  // namespace svq
