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
