"""B200 (sm_100a) implementation of the RWKV time-mixing WKV operator.

The operator is the per-channel decayed weighted mean of "Linear attention
without writing a CUDA kernel", section "The recurrence", carried as a
(numerator, denominator, max_exponent) state. The work runs in libwkv.so
(hand-written CUDA, C ABI in include/wkv.h); this package is its Python
binding:

    out, state = wkv_recurrence_b200.forward(k, v, w, u, state=None)
    out, state = wkv_recurrence_b200.forward_host(k_host, v_host, w, u)  # k, v in host memory
    out, state = wkv_recurrence_b200.step(state, k, v, w, u)

Importing the package does not load the library; the first call does, and
fails loudly if it is missing or no CUDA device is present.
"""

from .api import (WKV, PreparedForward, PreparedStep, WkvError, backward, empty_state, forward,  # noqa: F401
                  forward_host, forward_host_buffer_size, forward_kernel, forward_launches, make_workspace,
                  query_status, step, v6_forward, workspace_size)

__all__ = ["forward", "forward_host", "forward_host_buffer_size", "step", "backward", "WKV", "v6_forward",
           "workspace_size", "forward_kernel", "forward_launches", "make_workspace", "query_status", "empty_state",
           "PreparedForward", "PreparedStep", "WkvError"]
