#include "common.cuh"
#include "kernels.h"
namespace csa {
csa_status launch_attn_tc(const AttnArgs&, int, int, void*, size_t, cudaStream_t) { return CSA_ERR_UNSUPPORTED; }
size_t attn_tc_workspace_bytes(int, int, int, int, int, int, int, int) { return 0; }
}
