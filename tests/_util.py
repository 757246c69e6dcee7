"""Test helpers: convert synthetic workloads into the oracle's numpy inputs."""
import numpy as np
import torch

import oracle


def storage(t: torch.Tensor) -> np.ndarray:
    """Stored numbers as the oracle takes them: bfloat16 -> uint16 bits, float32 as is."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float32:
        return t.numpy()
    raise TypeError(t.dtype)


def oracle_tree(w) -> oracle.Tree:
    sh = w.shape
    return oracle.Tree(storage(w.root_keys), storage(w.mid_keys), storage(w.leaf_keys),
                       storage(w.leaf_values), sh.fanout,
                       None if w.root_child is None else w.root_child.cpu().numpy(),
                       None if w.mid_child is None else w.mid_child.cpu().numpy())


def oracle_inputs(w):
    return dict(q_kg=storage(w.q_kg), q_seq=storage(w.q_seq), k_seq=storage(w.k_seq), v_seq=storage(w.v_seq))
