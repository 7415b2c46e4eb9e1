"""Host-side layout of the LoRA parameters (CPU only): every A and B of every
linear of every layer has its own view into the flat fp32 / bf16 buffers,
starting on a 64-element boundary (128 bytes of the bf16 operand copy, so the
kernels' 16-byte TMA alignment holds), with the right shape, and no two views
overlap."""
import pytest
import torch

import synthetic as S


@pytest.mark.parametrize("name", ["tiny", "tiny-untied", "smollm2-135m", "llama-3.1-8b"])
def test_lora_views_aligned_disjoint_and_shaped(name):
    from nf4_layer_streamed_blockwise_b200.trainer import LoraParams
    sh = S.SHAPES[name]
    lp = LoraParams(sh, device="meta")
    spans = []
    for l in range(sh.n_layers):
        for n, (rows, cols) in sh.linear_shapes().items():
            for ab, shape in (("A", (sh.r, cols)), ("B", (rows, sh.r))):
                off, shp = lp.offsets[l][n][ab]
                assert tuple(shp) == shape
                assert off % 64 == 0
                spans.append((off, off + shape[0] * shape[1]))
                assert tuple(lp.view(lp.op, l, n, ab).shape) == shape
    spans.sort()
    assert all(a[1] <= b[0] for a, b in zip(spans, spans[1:]))
    assert spans[-1][1] <= lp.numel
    want = sh.n_layers * sum(sh.r * (rows + cols) for rows, cols in sh.linear_shapes().values())
    assert want <= lp.numel < want + 64 * len(spans)
    for buf, dt in ((lp.master, torch.float32), (lp.grad, torch.float32), (lp.m, torch.float32),
                    (lp.v, torch.float32), (lp.op, torch.bfloat16)):
        assert buf.dtype == dt and buf.numel() == lp.numel
