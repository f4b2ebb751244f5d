"""CPU oracle for the BASA forward path. Test infrastructure only: see basa_oracle."""
from .basa_oracle import (  # noqa: F401
    Geometry,
    attention_rows,
    basa_attention,
    cyclic_shift,
    dense_masked_attention,
    inverse_cyclic_shift,
    pool_kv,
    round_to_bf16,
    route_windows,
    to_grid,
    window_means,
    window_of_token,
    window_partition,
    window_unpartition,
)
