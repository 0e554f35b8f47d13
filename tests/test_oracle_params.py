"""Oracle pin: parameter accounting against the counts printed on the pages."""
from conftest import read_golden
from oracle.moe_oracle import MoEShape, param_counts

V3 = MoEShape(dim=7168, n_routed_experts=256, n_expert_groups=8, n_limited_groups=4,
              n_activated_experts=8, moe_inter_dim=2048)


def test_counts_match_pages():
    g = {k: int(v[0]) for k, v in read_golden("param_counts.txt").items()}
    c = param_counts(V3)
    for key in ("router", "routed_expert", "all_routed", "shared_expert", "block",
                "used_per_token"):
        assert c[key] == g[key], key
    assert c["block"] * 58 == g["block_x58"]
    assert c["router"] * 58 == g["router_x58"]
    assert V3.dim * V3.n_routed_experts == g["router_scores"]
    assert V3.n_routed_experts == g["router_bias"]
    assert g["router_scores"] + g["router_bias"] == g["router"]


def test_no_bias_router_count():
    # the bias exists only at dim 7168 in the gate-init excerpt; without it the
    # router is the score matrix alone
    s = MoEShape(dim=256, n_routed_experts=16, n_expert_groups=4, n_limited_groups=2,
                 n_activated_experts=4, moe_inter_dim=128, has_bias=False)
    assert param_counts(s)["router"] == 256 * 16
