// k2_state_scan.cu - the forward/backward scan of the state-build partials
// (scan.cuh) as a kernel of its own: one thread per unit.  The whole call runs
// the same scan inside the softmax kernel's otherwise idle warps; this launch
// serves the step-by-step interface and the export of the states after a call.
#include "kernels.h"
#include "scan.cuh"

namespace vdn {

namespace {
constexpr int kScanThreads = 128;
}

__global__ void __launch_bounds__(kScanThreads) k2_state_scan(const __grid_constant__ ScanArgs sa) {
  scan_range(sa, (long long)blockIdx.x * blockDim.x + threadIdx.x, (long long)gridDim.x * blockDim.x);
}

cudaError_t launch_state_scan(const ScanArgs& sa, cudaStream_t st) {
  const long long units = scan_units(sa.g);
  const long long blocks = (units + kScanThreads - 1) / kScanThreads;
  k2_state_scan<<<(unsigned)blocks, kScanThreads, 0, st>>>(sa);
  return cudaGetLastError();
}

}  // namespace vdn
