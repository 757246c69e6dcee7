"""The allocation-free entry point, atlaskv_attend_static.

It serves callers that cannot give the library device memory (a host program
that only speaks the C ABI and has no device allocator, a process whose device
memory another runtime has already partitioned, a hot loop where allocating is
not allowed): the scratch comes from a static array inside the library.  Its
results must match atlaskv_attend with a caller workspace, call after call.
This file is collected last on purpose.
"""
import ctypes

import pytest
import torch

from hierarchical_kv_pruning_b200 import binding, synth

pytestmark = pytest.mark.gpu


def _io(w, out, lse, kept):
    sh = w.shape
    return binding.atlaskv_io(sh.batch, sh.n_tokens, sh.n_heads, sh.seq_len, w.q_kg.data_ptr(),
                              w.q_seq.data_ptr(), w.k_seq.data_ptr(), w.v_seq.data_ptr(), out.data_ptr(),
                              lse.data_ptr(), kept[0].data_ptr(), kept[1].data_ptr(), kept[2].data_ptr())


def _outputs(w):
    sh = w.shape
    out = torch.empty_like(w.q_kg)
    lse = torch.empty((sh.batch, sh.n_tokens, sh.n_heads), dtype=torch.float32, device=w.q_kg.device)
    kept = tuple(torch.empty((sh.batch, sh.n_heads, k), dtype=torch.int32, device=w.q_kg.device) for k in sh.keep)
    return out, lse, kept


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_static_scratch_matches_workspace_path(dtype):
    sh = synth.custom(dtype=dtype, n_heads=8, n_kv_heads=2, head_dim=128, fanout=(12, 10, 9), keep=(3, 5, 16),
                      batch=4, n_tokens=24, seq_len=70, permuted=True)
    w = synth.make_workload(sh, "cuda", 31)
    with binding.HikvpTree.from_workload(w) as tree:
        ref = tree.attend(w.q_kg, w.q_seq, w.k_seq, w.v_seq, sh.keep)
        tree.sync_status()
        stream = torch.cuda.current_stream().cuda_stream
        for _ in range(2):   # two calls in a row share the static scratch
            out, lse, kept = _outputs(w)
            binding.atlaskv_attend_static(tree.handle, tree.params(sh.keep), _io(w, out, lse, kept), stream)
            tree.sync_status()
            for name, got in zip(("kept_root", "kept_mid", "kept_leaf"), kept):
                assert torch.equal(got, ref[name]), name
            err = (out.double() - ref["out"].double()).abs().max().item()
            tol = 1e-5 * ref["out"].double().abs().max().item() if dtype == torch.float32 else 2e-2
            assert err <= tol
            assert (lse - ref["lse"]).abs().max().item() <= 1e-4


def test_static_scratch_allocates_nothing():
    # After one warm call (the first call on a device looks up the static
    # array's address, and the runtime may load the library's device code
    # then), further calls change neither the device's free memory nor torch's
    # allocation count.
    sh = synth.custom(dtype=torch.bfloat16, n_heads=8, n_kv_heads=2, head_dim=128, fanout=(12, 10, 9),
                      keep=(3, 5, 16), batch=4, n_tokens=24, seq_len=70, permuted=True)
    w = synth.make_workload(sh, "cuda", 33)
    with binding.HikvpTree.from_workload(w) as tree:
        out, lse, kept = _outputs(w)
        io = _io(w, out, lse, kept)
        params = tree.params(sh.keep)
        stream = torch.cuda.current_stream().cuda_stream
        binding.atlaskv_attend_static(tree.handle, params, io, stream)
        tree.sync_status()
        torch.cuda.synchronize()
        free0 = torch.cuda.mem_get_info()[0]
        allocs0 = torch.cuda.memory_stats().get("allocation.all.allocated", 0)
        for _ in range(3):
            binding.atlaskv_attend_static(tree.handle, params, io, stream)
        tree.sync_status()
        torch.cuda.synchronize()
        assert torch.cuda.mem_get_info()[0] == free0
        assert torch.cuda.memory_stats().get("allocation.all.allocated", 0) == allocs0


def test_static_scratch_rejects_sizes_above_its_maximum():
    # B * H * D * 4 bytes of token sums alone exceed the 16 MiB maximum.
    sh = synth.custom(dtype=torch.bfloat16, n_heads=32, n_kv_heads=8, head_dim=128, fanout=(4, 4, 4),
                      keep=(1, 1, 1), batch=1100, n_tokens=1, seq_len=1)
    w = synth.make_workload(sh, "cuda", 32)
    with binding.HikvpTree.from_workload(w) as tree:
        assert tree.workspace_size(sh.keep, sh.batch, 1, sh.n_heads, 1) > binding.ATLASKV_STATIC_SCRATCH_BYTES
        out, lse, kept = _outputs(w)
        lib = binding.load_library()
        st = lib.atlaskv_attend_static(ctypes.c_void_p(tree.handle), ctypes.byref(tree.params(sh.keep)),
                                       ctypes.byref(_io(w, out, lse, kept)),
                                       ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == binding.ATLASKV_ENOMEM
        assert "static maximum" in binding.atlaskv_last_error()
