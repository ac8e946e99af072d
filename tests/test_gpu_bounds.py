"""The parity cases again, on the bounds-checked build of the library.

In place of a memory checker, the library's sources built with
SV_DEBUG_BOUNDS check every global index the kernels form -- the logit
range of every chunk and gather, workspace slots, list entries, tokens and
outputs -- against the extent of its buffer; a violation raises
SV_FLAG_BOUNDS in the workspace's status word and the access is skipped.
Here the GPU parity tests' own functions run on that build (ragged and
unaligned rows, strided and stride-0 views, invalid tokens and parents, the
early-exit batches, trees, every mode) and every workspace they used must
end with the bit clear, besides their own result checks passing.
"""
import numpy as np
import pytest
import torch

import speculative_decoding_verification_88_b200 as sv
from speculative_decoding_verification_88_b200 import build as svbuild

import test_gpu_parity as tp

pytestmark = pytest.mark.gpu

# greedy and multi-candidate cases run on both of their paths (one grid of
# row-chunk blocks, the persistent pipeline)
ARGMAX_CASES = [
    (tp.test_greedy_parity_shapes, dict(dtype="bf16", B=129, k=4, V=7)),
    (tp.test_greedy_parity_shapes, dict(dtype="f32", B=3, k=32, V=31)),
    (tp.test_greedy_parity_shapes, dict(dtype="bf16", B=1, k=8, V=4097)),
    (tp.test_greedy_parity_shapes, dict(dtype="bf16", B=2, k=4, V=128256)),
    (tp.test_greedy_parity_shapes, dict(dtype="f32", B=1, k=0, V=1)),
    (tp.test_greedy_strided_unaligned_and_broadcast, {}),
    (tp.test_greedy_early_exit_is_exact_and_leaves_the_workspace_clean,
     dict(B=512, k=8, V=32000, p_match=0.5)),
    (tp.test_greedy_invalid_drafts_raise_the_flag, {}),
    (tp.test_multi_parity_shapes, dict(dtype="bf16", B=2, G=64, k=3, V=50)),
    (tp.test_multi_parity_shapes, dict(dtype="f32", B=4, G=5, k=32, V=40)),
    (tp.test_multi_early_exit_is_exact_and_leaves_the_workspace_clean,
     dict(B=64, G=8, k=4, V=32000)),
    (tp.test_multi_rows_parity_shapes, dict(dtype="bf16", B=3, G=6, k=5, V=20480 + 17)),
    (tp.test_multi_rows_invalid_entries_and_limits, {}),
]
CASES = [(fn, dict(kw, argmax_path=path)) for fn, kw in ARGMAX_CASES
         for path in ("oneshot", "persistent")] + [
    (tp.test_threshold_invalid_tokens_and_workspace, {}),
    (tp.test_tree_invalid_parent_flag, {}),
    (tp.test_stochastic_parity_shapes, dict(t_dtype="bf16", d_dtype="f32", B=129, k=4, V=7,
                                            T=0.7)),
    (tp.test_stochastic_parity_shapes, dict(t_dtype="f32", d_dtype="bf16", B=3, k=32, V=33,
                                            T=1.0)),
    (tp.test_stochastic_parity_shapes, dict(t_dtype="bf16", d_dtype="bf16", B=3, k=8, V=4097,
                                            T=1.0)),
    (tp.test_stochastic_parity_shapes, dict(t_dtype="f32", d_dtype="f32", B=2, k=3, V=128256,
                                            T=1.0)),
    (tp.test_stochastic_parity_shapes, dict(t_dtype="bf16", d_dtype="f32", B=1, k=1, V=1,
                                            T=1.0)),
    (tp.test_stochastic_zero_drafts_samples_bonus, {}),
    (tp.test_stochastic_neg_inf_logits, {}),
    (tp.test_stochastic_strided_unaligned_views, {}),
    (tp.test_stochastic_invalid_token_and_residual_fallback, {}),
    (tp.test_stochastic_seq_offset_and_repeat, {}),
    (tp.test_tree_stochastic_parity_shapes, dict(dtype="bf16", B=4, N=64, V=40, T=1.3)),
    (tp.test_tree_stochastic_parity_shapes, dict(dtype="f32", B=2, N=33, V=2 * 16384 + 9,
                                                 T=1.0)),
    (tp.test_tree_stochastic_strided_unaligned_and_broadcast, {}),
    (tp.test_tree_stochastic_flags_and_clean_workspace, {}),
    (tp.test_one_workspace_across_modes_and_sizes, {}),
]


@pytest.fixture(scope="module")
def bounds_lib():
    path = svbuild.build(bounds=True)
    svbuild.build()
    return sv.load_library(path)


@pytest.mark.parametrize("fn,kw", CASES, ids=[f"{c[0].__name__}-{i}" for i, c in enumerate(CASES)])
def test_parity_case_on_the_bounds_checked_build(bounds_lib, monkeypatch, fn, kw):
    dev = torch.device("cuda:0")
    made = []
    init = sv.Workspace.__init__

    def recording_init(self, *a, **k):
        init(self, *a, **k)
        made.append(self)

    if "argmax_path" in kw:
        monkeypatch.setenv("SV_ONESHOT_MAX_BYTES",
                           "0" if kw["argmax_path"] == "persistent" else str(1 << 62))
    monkeypatch.setattr(sv, "_lib", bounds_lib)
    monkeypatch.setattr(sv, "_default_ws", {})
    monkeypatch.setattr(sv.Workspace, "__init__", recording_init)
    fn(dev, **kw)
    torch.cuda.synchronize()
    assert made, "the case used no workspace"
    for ws in made:
        if ws.buf is None:
            continue
        flags = ws.device_status(clear=False)
        line = int(ws.buf[20:24].cpu().numpy().view(np.uint32)[0])
        assert not flags & sv.SV_FLAG_BOUNDS, f"bounds violation at sv source line {line}"
