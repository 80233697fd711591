"""CPU oracle for LoSA's hot path (test infrastructure only).

Imported only by the tests, the smoke check and the benchmark's CPU
baseline leg; the library itself never imports it.
"""
from .losa_oracle import (FX_ONE, attention_rows, attention_probs, block_mass,
                          block_mass_row, dense_attention, retained_keys, select,
                          select_row, sparse_attention, sparse_attention_block,
                          tau_fixed, to_fixed)
