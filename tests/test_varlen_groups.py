"""The launch groups of sa_attn_fwd_varlen, host logic only (no GPU): sequences are taken
longest first, and a group takes the next sequence while its heads padded to the group's
longest sequence stay within twice their own padded size, or below 2^20 padded token-heads,
and its heads stay at most 65535.  Checked as properties of the rule, on random and on the
edge-case batches."""
import numpy as np
import pytest


def _pad(n):
    return -(-n // 128) * 128


def _admits(members, H):
    """The group rule for members (lengths, longest first): every prefix that adds a member
    keeps the padded size within twice its own or under 2^20 padded token-heads, and the
    group's heads at most 65535."""
    pmax = _pad(members[0])
    own = pmax
    for k, n in enumerate(members[1:], start=1):
        own += _pad(n)
        pad = (k + 1) * pmax
        if pad > 2 * own and pad * H > (1 << 20):
            return False
        if (k + 1) * H > 65535:
            return False
    return True


def _check(libsa, lens, H):
    g = libsa.sa_debug_varlen_groups(lens, H)
    n = max(g) + 1
    assert sorted(set(g)) == list(range(n))
    # launch order: longest first; within equal lengths, the original order
    order = sorted(range(len(lens)), key=lambda i: (-lens[i], i))
    assert [g[i] for i in order] == sorted(g)
    groups = [[lens[i] for i in order if g[i] == k] for k in range(n)]
    for k, members in enumerate(groups):
        assert _admits(members, H), (k, members)
        if k + 1 < n:  # maximal: the next group's first sequence would break the rule
            assert not _admits(members + [groups[k + 1][0]], H), (k, members)
    return groups


def test_short_sequences_form_one_group(libsa):
    lens = [int(n) for n in np.random.default_rng(77).integers(1, 513, size=64)]
    assert len(_check(libsa, lens, 2)) == 1


def test_one_long_and_many_short_sequences(libsa):
    groups = _check(libsa, [40000] + [1000] * 40, 1)
    assert [len(m) for m in groups] == [26, 15]


@pytest.mark.parametrize("seed", range(6))
def test_random_batches(libsa, seed):
    rng = np.random.default_rng(seed)
    nseq = int(rng.integers(1, 200))
    lens = [int(x) for x in np.exp(rng.uniform(0, np.log(200000), size=nseq)).astype(int) + 1]
    _check(libsa, lens, int(rng.choice([1, 2, 12, 40])))


def test_head_limit(libsa):
    # 65535 heads: every sequence alone; 32768 heads: at most one per group as well
    assert libsa.sa_debug_varlen_groups([10, 10, 10], 65535) == [0, 1, 2]
    assert len(_check(libsa, [5] * 7, 32768)) == 7
    # 40 heads: at most 1638 short sequences per group
    assert [len(m) for m in _check(libsa, [3] * 2000, 40)] == [1638, 362]


def test_bad_arguments(libsa):
    with pytest.raises(ValueError):
        libsa.sa_debug_varlen_groups([], 2)
    with pytest.raises(ValueError):
        libsa.sa_debug_varlen_groups([5, 0], 2)
    with pytest.raises(ValueError):
        libsa.sa_debug_varlen_groups([5], 0)
