"""DeepSeek Sparse Attention (DSA) forward path for NVIDIA B200 (sm_100a).

Three stages, each a hand-written CUDA kernel behind a C ABI (``libdsa.so``,
declared in ``include/dsa.h``):

  indexer_scores   I[t,s] = sum_j w[t,j] * ReLU(q^I[t,j] . k^I[s]), s <= t
  topk             S_t = the k largest I[t,s], ties to the lower s
  sparse_attn      softmax attention of every query head over S_t
  forward          the three back to back on one stream
  indexer_kl       the indexer's training loss KL(p_t || Softmax(I_t)) and
                   its gradient with respect to the scores
  indexer_backward dq, dk, dw of the indexer inputs for that gradient

The Python functions are argument marshalling only; every step runs in the
CUDA library, which is loaded on first use and raises if it is missing.
"""
from .inputs import WORKLOADS, Workload, make_inputs, to_device  # noqa: F401


_BINDING_NAMES = ("indexer_scores", "topk", "sparse_attn", "forward", "forward_args",
                  "forward_workspace_bytes", "attn_shape", "load_library", "DSAError", "device_error",
                  "kernel_launch_count", "indexer_kl", "indexer_backward")


def __getattr__(name):
    # The binding loads libdsa.so on first call; it is imported lazily so that
    # CPU-only users of the input generator do not need the CUDA library.
    if name in _BINDING_NAMES:
        import importlib
        return getattr(importlib.import_module(".binding", __name__), name)
    raise AttributeError(name)
