"""Seeded synthetic inputs shared by the oracle tests, the GPU tests and the bench."""
from .synthetic import (CONFIGS, SWEEP_N, Workload, clustered_pair, gaussian_pair, generate,
                        get_config, rope_rotate, sweep_config, tiny_custom, unit_list)
from .chain import CHAIN_CONFIGS, ChainWorkload, generate_chain, relation_workload

__all__ = ["CONFIGS", "SWEEP_N", "Workload", "clustered_pair", "gaussian_pair", "generate", "get_config",
           "rope_rotate", "sweep_config", "tiny_custom", "unit_list",
           "CHAIN_CONFIGS", "ChainWorkload", "generate_chain", "relation_workload"]
