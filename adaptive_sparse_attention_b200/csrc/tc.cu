// tc.cu -- tensor-core (tcgen05) kernels of the entmax attention forward pass, bf16.
// Placeholder launchers until the tcgen05 kernels land: they run the CUDA-core kernels.
#include "kernels.h"

namespace ea {

cudaError_t launch_tau_tc(const Problem& P, cudaStream_t s) { return launch_tau_simt(P, 1, s); }
cudaError_t launch_out_tc(const Problem& P, cudaStream_t s) { return launch_out_simt(P, 1, s); }

}  // namespace ea
