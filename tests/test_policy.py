"""fused_qk_norm_rope_min_tokens: the page's rules, one by one
("vllm_omni.diffusion.layers.fused_qk_norm_rope", fused_qk_norm_rope_min_tokens)."""
import pytest

from qk_rmsnorm_rope_qknr_b200 import policy


@pytest.fixture
def env(monkeypatch):
    monkeypatch.delenv(policy.ENV_MIN_TOKENS, raising=False)
    return monkeypatch


def test_unset_gives_default(env):
    assert policy.fused_qk_norm_rope_min_tokens(2048) == 2048


@pytest.mark.parametrize("blank", ["", " ", "\t\n"])
def test_blank_gives_default(env, blank):
    env.setenv(policy.ENV_MIN_TOKENS, blank)
    assert policy.fused_qk_norm_rope_min_tokens(2048) == 2048


@pytest.mark.parametrize("text,want", [("0", 0), ("4096", 4096), (" 17 ", 17), ("00012", 12)])
def test_integers_override(env, text, want):
    env.setenv(policy.ENV_MIN_TOKENS, text)
    assert policy.fused_qk_norm_rope_min_tokens(2048) == want


@pytest.mark.parametrize("bad", ["-1", "1.5", "abc", "12a", "+5", "1e3", "0x10"])
def test_anything_else_raises(env, bad):
    env.setenv(policy.ENV_MIN_TOKENS, bad)
    with pytest.raises(ValueError):
        policy.fused_qk_norm_rope_min_tokens(2048)


def test_read_at_call_time(env):
    assert policy.should_fuse(1000, 2048) is False
    env.setenv(policy.ENV_MIN_TOKENS, "0")          # 0 = always fuse
    assert policy.should_fuse(1, 2048) is True
    env.setenv(policy.ENV_MIN_TOKENS, "5000")
    assert policy.should_fuse(4096, 2048) is False
    env.delenv(policy.ENV_MIN_TOKENS)
    assert policy.should_fuse(4096, 2048) is True
