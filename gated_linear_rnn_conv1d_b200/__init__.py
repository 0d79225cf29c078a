"""B200-native RG-LRU temporal core: Conv1D(4) → RG-LRU, prefill scan and decode step."""
