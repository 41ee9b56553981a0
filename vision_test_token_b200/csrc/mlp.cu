// mlp.cu -- placeholder until the MLP kernels land.
#include "ttt_internal.h"
namespace ttt {
size_t mlp_ws_bytes(const ttt_shape&) { return kWsHeader; }
ttt_status launch_mlp(const Call&) { return TTT_ERR_UNSUPPORTED; }
}  // namespace ttt
