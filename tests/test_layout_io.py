"""Placements and statistics round-trip through save_layout / load_layout
(the checkpoint of a re-layout: placement, rank scores, replicas, counts)."""
import numpy as np


def test_layout_round_trip(tmp_path, orc):
    from co_activation_placement_b200 import pipeline
    rng = np.random.default_rng(0)
    E, G, rpn, L = 16, 4, 2, 3
    ids = np.stack([np.stack([rng.permutation(E)[:3] for _ in range(200)]) for _ in range(L)]).astype(np.int32)
    st = orc.coact(ids, E)
    e2r = [orc.place_correlated(st["coact"][l], G, rpn) for l in range(L)]
    rs = [orc.rank_score(st["trans"][l], e2r[l + 1], G) for l in range(L - 1)]
    reps = [orc.place_replicas(st["coact"][l], G, rpn, e2r[l], 1) for l in range(L)]
    path = str(tmp_path / "layout.npz")
    pipeline.save_layout(path, e2r, rs, reps, stats=st)
    back = pipeline.load_layout(path)
    assert all((a == b).all() for a, b in zip(back["expert_to_rank"], e2r))
    assert all((a == b).all() for a, b in zip(back["rank_score"], rs))
    assert all((a[0] == b[0]).all() and (a[1] == b[1]).all() for a, b in zip(back["replicas"], reps))
    assert (back["stats"]["coact"] == st["coact"]).all() and (back["stats"]["trans"] == st["trans"]).all()
    assert back["stats"]["ochiai"].dtype == np.float32


def test_layout_minimal(tmp_path):
    from co_activation_placement_b200 import pipeline
    path = str(tmp_path / "l.npz")
    pipeline.save_layout(path, [np.arange(8, dtype=np.int32) // 2])
    back = pipeline.load_layout(path)
    assert back["rank_score"] == [] and back["replicas"] == [] and back["stats"] == {}
    assert back["expert_to_rank"][0].tolist() == [0, 0, 1, 1, 2, 2, 3, 3]
