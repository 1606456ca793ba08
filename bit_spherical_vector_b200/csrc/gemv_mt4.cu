// gemv_mt4.cu -- GEMV kernel instantiation for 4 token(s) per pass
// (one translation unit per batch width so the builds run in parallel).
#include "gemv_impl.cuh"

namespace svq {
template cudaError_t launch_gemv_mt<4>(const GemvKParams&, int, size_t, cudaStream_t);
}  // namespace svq
