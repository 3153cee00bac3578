"""B200-native KnapSpec knapsack layer-selection DP.

The compute path lives in the C-ABI library ``libknapspec.so`` (hand-written
CUDA for sm_100a); :mod:`knapsack_layer_selection_b200.binding` marshals
arguments to it.  :mod:`knapsack_layer_selection_b200.workloads` describes the
synthetic workloads and draws their seeded inputs.  Importing the package does
not load the library; the binding loads it on first use and raises if it is
missing.
"""
