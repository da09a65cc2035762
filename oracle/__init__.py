"""CPU oracle for the LoLA chunkwise hybrid-attention path.

TEST INFRASTRUCTURE ONLY: imported by tests/, __graft_entry__.smoke() and the
cpu_baseline / reference leg of bench.py, never by the product library.
"""
from .lola_oracle import (LolaStream, feature_map, self_recall_error, top_lambda,
                          valid_alternative, state_elements, full_elements, sre_map, TIE_REL,
                          HIDE_STATE, HIDE_SPARSE, SCORERS)

__all__ = ["LolaStream", "feature_map", "self_recall_error", "top_lambda",
           "valid_alternative", "state_elements", "full_elements", "sre_map", "TIE_REL",
           "HIDE_STATE", "HIDE_SPARSE", "SCORERS"]
