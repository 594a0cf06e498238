"""B200-native Medusa draft-and-verify step: CUDA kernels (sm_100a) behind a
C ABI (include/medusa.h), with a thin PyTorch binding in ``api``."""
from .api import (Tree, device_status, medusa_accept_greedy, medusa_accept_typical,  # noqa: F401
                  medusa_build_tree, medusa_heads_forward, medusa_kv_compact, medusa_topk,
                  medusa_tree_attention, tree_plan_host, version)
