#include "cowa_internal.h"
namespace cowa {
size_t bwd_workspace_bytes(int B, int N, int Hq, int Hkv, int d) { return (size_t)B * Hq * N * 4; }
cudaError_t launch_bwd(const BwdArgs& a, cudaStream_t s) { return cudaErrorNotSupported; }
}
