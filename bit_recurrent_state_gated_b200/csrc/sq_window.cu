// sq_window.cu -- windowed variant (requantize every W tokens); not built yet.
#include "sq_internal.h"

namespace sq {
cudaError_t launch_window_step(const StepArgs&, int, int, int, cudaStream_t) {
  return cudaErrorNotSupported;
}
cudaError_t launch_window_flush(const StepArgs&, int, cudaStream_t) {
  return cudaErrorNotSupported;
}
}  // namespace sq
