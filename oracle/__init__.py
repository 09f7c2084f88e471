"""CPU oracle for the Block Transformer inference path (test infrastructure).

Only the test suite, the smoke check and the benchmark's CPU-baseline leg
import this package; the product path never does.
"""
from .model import (BlockTransformerOracle, OracleSession, attend,  # noqa: F401
                    embed_blocks, gelu, layer_norm, prefix_projection,
                    pythia_layer, rotary)
