"""vision_test_token_b200 -- B200-native (sm_100a) forward pass of the ViT^3 test-time-training
(TTT) token-mixing layer.

The compute lives in ``libttt.so`` (CUDA kernels behind the C ABI of ``include/ttt.h``); this
package holds its ctypes binding (``capi``), torch-facing wrappers (``layer``), the seeded input
generator (``inputs``) and the build script (``build``).
"""
from .inputs import WORKLOADS, Workload, make_inputs  # noqa: F401
from .layer import (backward_dwconv, backward_linear, backward_mlp, forward_conv3x3, forward_dwconv, forward_layer, forward_linear,  # noqa: F401
                    forward_linear_minibatch, forward_mlp, workspace, workspace_status)

__all__ = ["WORKLOADS", "Workload", "make_inputs", "forward_linear", "forward_linear_minibatch", "forward_dwconv",
           "forward_conv3x3", "forward_mlp", "forward_layer", "backward_linear", "backward_dwconv", "backward_mlp", "workspace", "workspace_status"]
