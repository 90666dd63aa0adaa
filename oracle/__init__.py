"""CPU oracle for the AdaSpark layer hot path -- TEST INFRASTRUCTURE ONLY.

Plain, slow numpy code in float64 that states what the path computes, one
function per step, each citing the passage of the AdaSpark pages it follows.
It shares no code with the CUDA library (``ffn_long_video_b200``) and neither
imports the other.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may use it; the
product path never routes through it.

Parity status per function (what pins it is in ``tests/test_oracle_pins.py``):

* ``cube_partition``        pinned (brute-force sort order on small grids)
* ``cube_mean_keys``        pinned (invariants: zero residual sum, constant cubes)
* ``top_p``                 pinned (exhaustive subset enumeration, closed forms)
* ``top_k``                 pinned (exhaustive k-subset enumeration, closed forms)
* ``uniform_cubes``, ``select_cubes_uniform``
                            pinned (hand values, even-spacing and count
                            invariants, equal sets across heads and tokens)
* ``select_cubes``          pinned (uniform closed form, 2-cube sigmoid cut, GQA map)
* ``attention_given_sets``  pinned (torch SDPA in float64 with a mask; first token)
* ``ffn_select``            pinned (closed forms on scaled tokens, brute force)
* ``token_importance``      pinned (closed forms for the three normalisations)
* ``linear``, ``rmsnorm``   pinned (explicit loops; closed forms and invariances)
* ``swiglu_ffn``            pinned (torch.nn.functional in float64)
* ``token_ffn``             pinned (p=1 dense, compensation identity, text rows)
* ``attention_backward_given_sets``, ``swiglu_ffn_backward``,
  ``ffn_backward_given_sets``
                            pinned (full central-difference Jacobians of the
                            pinned forward functions; torch autograd in float64
                            on the dense cases; sum invariants)
* agreement with the authors' own numbers: parity unpinned (the pages print
  no worked example for any step; see the module docstring of adaspark_ref).
"""
from .adaspark_ref import (  # noqa: F401
    cube_partition,
    cube_mean_keys,
    cube_scores,
    softmax,
    top_p,
    top_p_margin,
    top_k,
    top_k_margin,
    select_cubes,
    select_cubes_uniform,
    uniform_cubes,
    token_importance,
    linear,
    rmsnorm,
    attention_given_sets,
    cube_attn,
    ffn_select,
    swiglu_ffn,
    ffn_given_sets,
    token_ffn,
    attention_backward_given_sets,
    swiglu_ffn_backward,
    ffn_backward_given_sets,
)
