"""CPU fp64 oracle for the KDA token mixer (test infrastructure only)."""
from .kda_oracle import (kda_recurrence, kda_chunked, short_conv, l2norm, output_gate,  # noqa: F401
                         kda_mixer, kda_decode_step, kda_decode_steps, token_step)
