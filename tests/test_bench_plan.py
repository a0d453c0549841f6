"""Host-side bookkeeping of bench.py on CPU: the launch plan it reports where steps are
not CUDA graphs (on graph-replayed steps it counts the graphs' kernel nodes instead, and
the two agree on every workload), and the graceful fallback of the graph inspection."""
import dataclasses
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import bench  # noqa: E402
from cross_layer_compressed_b200 import synth  # noqa: E402


def test_rank_space_launch_plan():
    # dense 128K at batch 1: 147 spans per head -> merge and projection in one kernel
    assert bench._ra_kernels(synth.LLAMA8B_DENSE_128K, 0) == 3
    # dense at batch 8: 18 spans per sequence -> separate merge and projection
    assert bench._ra_kernels(dataclasses.replace(synth.LLAMA8B_DENSE_128K, batch=8), 0) == 4
    # selective 32K (261 chunks of 8 rows = 9 items of <= 256 rows) and 16K
    w = synth.LLAMA8B_SR_32K
    assert bench._ra_kernels(w, w.n_sel) == 4
    w = synth.QWEN14B_SR_16K
    assert bench._ra_kernels(w, w.n_sel) == 4
    # many selected chunks: 32 or more items per head take the fused kernel
    w = synth.LLAMA8B_SR_32K
    assert bench._ra_kernels(w, 1024) == 3         # 8192 rows -> 32 items


def test_graph_inspection_falls_back_to_none():
    class NotAGraph:
        def raw_cuda_graph(self):
            raise RuntimeError("no graph")
    assert bench.count_kernel_nodes(NotAGraph()) is None
