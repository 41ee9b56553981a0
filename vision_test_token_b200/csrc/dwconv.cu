// dwconv.cu -- placeholder until the depthwise-conv kernels land.
#include "ttt_internal.h"
namespace ttt {
size_t dwconv_ws_bytes(const ttt_shape&) { return kWsHeader; }
ttt_status launch_dwconv(const Call&) { return TTT_ERR_UNSUPPORTED; }
}  // namespace ttt
