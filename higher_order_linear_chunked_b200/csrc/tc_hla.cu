// tcgen05 walker kernels (placeholder until the walkers land): nothing is routed here yet.
#include "tc.h"

namespace hla {
namespace tc {

bool supported(int, bool, bool, int) { return false; }
size_t workspace_bytes(int, bool, int, int) { return 0; }
int kernel_launches(int, bool, int, int) { return 0; }
cudaError_t forward(int, bool, const void*, const void*, const void*, float, float*, int, int, void*, int*,
                    cudaStream_t, cudaEvent_t*) {
    return cudaErrorNotSupported;
}

}  // namespace tc
}  // namespace hla
