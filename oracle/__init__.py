"""Float64 CPU oracle for the Infini-attention layer forward pass.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library, its
Python binding, the package) imports, calls or links anything in this folder.
Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may use it.

The oracle shares no code with the CUDA path.  Both sides consume the same
seeded inputs, produced by ``compressive_memory_transformer_segment_b200.synth``,
which holds none of the method's arithmetic.

Pinned functions (each is checked in ``tests/test_oracle_pins.py`` against a
library routine, a closed form, brute force or an invariant):
  elu_plus_one, gate_sigmoid, local_causal_attention, memory_retrieval,
  memory_update (linear and delta), infini_attention_forward, scan_states,
  segment_output.
The backward (``infini_backward``: elu_plus_one_grad, the vector-Jacobian
products of each step and infini_attention_backward) is pinned in
``tests/test_oracle_backward.py`` against central finite differences of the
forward and closed forms of special cases.
The prologue (``infini_projection``: rope_angles, rope_tables, apply_rope,
qkv_projection, qkv_project_rope) is pinned in
``tests/test_oracle_projection.py`` against brute-force loops, the complex
form of the rotation and its invariants.
No function here is "parity unpinned".
"""

from .infini_oracle import (  # noqa: F401
    elu_plus_one,
    gate_sigmoid,
    local_causal_attention,
    memory_retrieval,
    memory_update,
    segment_bounds,
    scan_states,
    segment_output,
    infini_attention_forward,
)
from .infini_backward import (  # noqa: F401
    elu_plus_one_grad,
    local_causal_attention_vjp,
    memory_retrieval_vjp,
    memory_update_vjp,
    segment_output_vjp,
    infini_attention_backward,
)
from .infini_projection import (  # noqa: F401
    rope_angles,
    rope_tables,
    apply_rope,
    qkv_projection,
    qkv_project_rope,
)
