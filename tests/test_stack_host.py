"""Host-side logic of the stack driver that needs no GPU."""
from compressed_sparse_attention_13_b200.stack import v4_pro_schedule


def test_v4_pro_layer_schedule():
    """61 layers: HCA at layers 0-1, then CSA and HCA alternating from layer 2
    (CSA first), then the MTP block with the sliding window only."""
    kinds = v4_pro_schedule()
    assert len(kinds) == 62 and kinds[-1] == "window"
    assert kinds[:2] == ["hca", "hca"]
    assert all(kinds[i] == ("csa" if i % 2 == 0 else "hca") for i in range(2, 61))
    assert kinds.count("csa") == 30 and kinds.count("hca") == 31
    assert v4_pro_schedule(mtp=False) == kinds[:61]


def test_layer_caches_are_sized_in_whole_128_row_steps():
    """A layer's pooled caches hold every block its tokens can complete, in
    whole 128-row steps (a capacity that is not a multiple of 4 would take
    the CSA layers off the tensor-core MXFP4 indexer); the raw window starts
    W - 1 tokens before the first new token (at it when W = 0).  Allocated
    on the CPU: the sizing is host logic."""
    from compressed_sparse_attention_13_b200 import params
    from compressed_sparse_attention_13_b200.stack import Layer, LayerSpec
    cases = [("csa", 4, 128, 1_044_480, 4096 + 256), ("hca", 128, 128, 1_044_480, 4096 + 256),
             ("csa", 4, 128, 4, 254), ("hca", 128, 128, 0, 200), ("csa", 4, 0, 8, 3), ("window", 4, 128, 0, 16)]
    for kind, m, W, prior, new in cases:
        p = params(m, W, 512, 64, 512, 64, 128, 512 ** -0.5)
        L = Layer(LayerSpec(kind, p, prior, new), device="cpu")   # the library gives the workspace size
        need = (prior + new) // m
        assert L.cap_blocks % 128 == 0 and need <= L.cap_blocks < need + 128
        if kind == "window":
            assert L.kv is None and L.kI is None
        else:
            assert L.kv.data.shape[0] == L.cap_blocks
            assert (L.kI is not None) == (kind == "csa")
        assert L.raw_pos0 == (prior - (W - 1) if W > 0 else prior)
        assert L.n_raw == max(W - 1, 0) + new and L.x.shape[0] == L.n_raw
        assert L.t_next == prior and L._pooled == -(-prior // m)
