"""Helpers shared by the GPU parity tests."""
import numpy as np

from fp4_kv_cache_03_b200 import synth


def small_workload(name="small", lengths=(4096,), q_per_seq=1, D=128, H=16, H_I=4, d_I=64,
                   topk=64, window=128, modes=("full",), pool_blocks=0, seed=11, ratio=1,
                   q_token0=(), append=False, outlier_frac=0.0):
    return synth.Workload(name, seed, len(lengths), tuple(int(v) for v in lengths), q_per_seq,
                          D, H, H_I, d_I, topk, window, tuple(modes), pool_blocks=pool_blocks,
                          ratio=ratio, q_token0=tuple(q_token0), append=append,
                          outlier_frac=outlier_frac)


def gpu_indices(dw, used):
    """The index tensors each layer used, as numpy int64 arrays [num_q, topk]."""
    return [u.cpu().numpy().astype(np.int64) for u in used]
