"""fp64 CPU oracle for GPTQ-2D (test infrastructure only; never used by the library)."""
from .gptq2d_oracle import *  # noqa: F401,F403
from .gptq2d_oracle import (NEAR_TIE_BAND, Result, babai_kron_sweep, closest_vector_exhaustive,
                            entry_value, gptq2d, gptq2d_antidiagonal, gptq_1d_obs, grid_bounds,
                            near_tie, nearest_plane_by_definition, proxy_loss, reverse_cholesky,
                            round_to_grid, rtn, sphere_decode)
from .gptq2d_oracle import (babai_tensor_sweep, gptq_kron_hyperplane, gptq_kron_via_2d,
                            kron_factor, kron_gram, mode_product, proxy_loss_tensor)
from .gptq2d_oracle import expand_grid, pack_nibbles, packed_codes, stored_codes
from .gptq2d_oracle import gram, gram_batches
