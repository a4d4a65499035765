"""Closed-form checks of the Beam layer shape against the figures the pages print.

Sources: 'Welcome Beam' page, section 'Mixture of Experts' (256 experts, SwiGLU intermediate
2,560, "about 39M parameters" each, experts hold 98.4% of the parameters, 49 MoE layers);
section 'Attention' (hidden 5,120); the reducer.xgoose.org digest page, section 'Multi-GPU and
multi-node' of the flattened post (8B replicated non-expert parameters); the aicoder.com
tech-report page, 'Key Takeaways' (501.3B total / 23.4B active).
"""
import beam_synth as bs


def test_beam_layer_shape_closed_forms():
    L = bs.WORKLOADS["prefill"].layer
    H, I, E, k = L["hidden"], L["inter"], L["n_experts"], L["topk"]
    assert (H, I, E, L["n_groups"], L["topk_groups"], k, L["group_topn"], L["routed_scale"]) == \
        (5120, 2560, 256, 8, 4, 8, 2, 2.5)
    per_expert = 3 * H * I
    assert per_expert == 39_321_600                      # "about 39M parameters"
    n_moe_layers = 49
    expert_params = n_moe_layers * E * per_expert
    non_expert = 8e9                                     # "8B parameters" replicated under EP
    total = expert_params + non_expert
    assert abs(expert_params / 1e9 - 493.25) < 0.01
    assert round(total / 1e9) == 501                     # "501B"
    assert abs(total / 1e9 - 501.3) < 0.1                # "501.3B"
    assert round(100 * expert_params / total, 1) == 98.4  # "98.4%"
    active = n_moe_layers * k * per_expert + non_expert
    assert round(active / 1e9) == 23                     # "23B active"
    assert abs(active / 1e9 - 23.4) < 0.05               # "23.4B active"
    # one layer's experts resident in bf16 (~20 GB)
    assert E * per_expert * 2 == 20_132_659_200


def test_every_workload_is_consistent():
    for wl in list(bs.WORKLOADS.values()) + list(bs.PARITY_CASES.values()):
        assert wl.n_experts % wl.n_groups == 0
        assert 1 <= wl.topk_groups <= wl.n_groups
        assert wl.topk <= wl.topk_groups * wl.n_experts // wl.n_groups
        assert wl.group_topn <= wl.n_experts // wl.n_groups
        assert wl.hidden % 64 == 0 and wl.inter % 64 == 0


def test_dense_intermediate_reading_matches_8b_non_expert():
    """I_dense = 20,480 (a reading) with the pages' attention shapes gives the '8B' non-expert count.

    Attention per layer: W_q 5120 x (48 x 128), W_k and W_v 5120 x (8 x 128), W_o (48 x 128) x 5120 and the
    sigmoid output gate 5120 x (48 x 128) ('Welcome Beam', section 'Attention'); 52 layers; vocabulary
    151,936 (tech-report page, 'Key Takeaways'), embeddings and LM head untied (reading); routers
    49 x 256 x 5120; 3 dense SwiGLU layers of intermediate size I.
    """
    H, q, kv = 5120, 48 * 128, 8 * 128
    attn = 52 * (H * q + 2 * H * kv + q * H + H * q)
    emb = 2 * 151_936 * H
    routers = 49 * 256 * H
    I = bs.DENSE["dense_prefill"].inter
    dense = 3 * 3 * H * I
    total = attn + emb + routers + dense
    assert I == 20480 and round(total / 1e9) == 8          # "8B parameters" replicated under EP
    assert abs(total / 1e9 - 8.0) < 0.05
