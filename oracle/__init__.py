"""CPU oracle of the flow-matching action head (fp64, numpy).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()`` and
the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py``.  The product
path (``flow_matching_dit_b200``) never imports it, and it never imports the
product.  See ``oracle/dit.py`` for the sources each function follows.
``oracle.grad`` (imported on its own: it needs torch) adds the gradients of
the training loss.
"""

from .dit import (Model, action_decoder, action_encoder, ada_layer_norm, attention,  # noqa: F401
                  category_linear, cross_key_mask, cross_kv, dit, dit_block, euler_schedule, gelu, get_action,
                  layer_norm, linear, prepare_sample, relu, silu, sinusoidal_embedding,
                  state_encoder, swish, timestep_embedding, to_f64, training_loss, velocity)
