"""FP64 CPU oracle (test infrastructure only; see gdn_oracle's header)."""
from .gdn_oracle import (as_f64, gdn_transition, gdn_transition_explicit, prefill, chains,
                         check_parents, full_state_decode, full_state_decode_states,
                         replay_decode, closed_form_state, decode_batch, ancestry_table)

__all__ = ["as_f64", "gdn_transition", "gdn_transition_explicit", "prefill", "chains",
           "check_parents", "full_state_decode", "full_state_decode_states", "replay_decode",
           "closed_form_state", "decode_batch", "ancestry_table"]
