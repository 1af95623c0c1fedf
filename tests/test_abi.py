"""The C ABI library loads, exports every entry point include/engram.h
declares, and its host-side checks answer without touching a GPU."""
import os
import re

import numpy as np

from hashed_gram_conditional_engram_b200 import engram as eg

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "engram.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(engram_[a-z_0-9]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    L = eg.lib()
    names = declared_symbols()
    assert len(names) >= 10
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(eg.EXPORTED)


def _cfg(**kw):
    a = dict(K=2, D_h=16, d_model=64, n_branch=1, V_raw=1000, V_c=770, dtype=eg.F32,
             rows=[1009] * 4, mult=np.ones((4, 3), np.uint64))
    a.update(kw)
    return eg.make_cfg(**a)


def test_workspace_sizes_host_only():
    c = _cfg()
    assert eg.engram_workspace_size(c, eg.WS_FORWARD, 64) > 0
    assert eg.engram_workspace_size(c, eg.WS_BACKWARD, 64) > eg.engram_workspace_size(
        c, eg.WS_TABLE_GRAD, 64)
    assert eg.engram_workspace_size(None, eg.WS_VOCAB, 129280) > 129280 * 8
    assert eg.engram_saved_size(c, 64) >= 64 * (1 + 3 * 64) * 4
    b = _cfg(K=8, D_h=80, d_model=2560, dtype=eg.BF16, rows=[4449997] * 16,
             mult=np.ones((16, 3), np.uint64))
    # bf16: gate partials (2 per 256-column tile per token), the gate itself and
    # the two counters of the one-launch decode step
    assert eg.engram_workspace_size(b, eg.WS_FORWARD, 32768) == 32768 * 20 * 16 + 32768 * 4 + 256
    assert eg.engram_saved_size(b, 32768) == 32768 * 4
    # keeping k and v: alpha up to the next 256 bytes, then fp32 [N, 2d]; the
    # backward then needs no room of its own for them
    bk = _cfg(K=8, D_h=80, d_model=2560, dtype=eg.BF16, rows=[4449997] * 16,
              mult=np.ones((16, 3), np.uint64), flags=eg.SAVE_KV)
    assert eg.engram_saved_size(bk, 1000) == 4096 + 1000 * 2 * 2560 * 4
    assert (eg.engram_workspace_size(b, eg.WS_BACKWARD, 32768)
            - eg.engram_workspace_size(bk, eg.WS_BACKWARD, 32768)) >= 32768 * 2 * 2560 * 4
    # fp32 layers keep their own intermediates and ignore the flag
    assert eg.engram_saved_size(_cfg(flags=eg.SAVE_KV), 64) == eg.engram_saved_size(c, 64)


def test_small_parameter_block_sizes():
    """conv weights [d, 4] or [M, d, 4], then g_h, g_k (and g_v) of [M, d]."""
    d, M = 64, 3
    for flags, want in [(0, 4 * d), (eg.CONV_DILATED | eg.CONV_PRENORM, 4 * d),
                        (eg.CONV_PER_BRANCH, 4 * d * M), (eg.NORM_SCALES, 4 * d + 2 * M * d),
                        (eg.NORM_SCALES | eg.CONV_PRENORM | eg.CONV_PER_BRANCH,
                         4 * d * M + 3 * M * d)]:
        assert eg.engram_param_floats(_cfg(n_branch=M, flags=flags)) == want, flags
    assert eg.engram_param_floats(_cfg(flags=64)) == 0  # not a flag: invalid configuration
    # bf16 layers (one branch): conv weights, then g_h, g_k, and g_v with the
    # pre-conv norm
    d = 256
    for flags, want in [(0, 4 * d), (eg.CONV_PRENORM, 4 * d), (eg.NORM_SCALES, 6 * d),
                        (eg.NORM_SCALES | eg.CONV_PRENORM | eg.CONV_DILATED, 7 * d)]:
        c = _cfg(d_model=d, K=2, D_h=32, dtype=eg.BF16, flags=flags)
        assert eg.engram_param_floats(c) == want, flags


def test_prenorm_workspace_holds_v_and_rc():
    """With the pre-conv norm a bf16 forward also needs v (fp32 [N, d]) and
    rc [N]; the backward dc (fp32 [N, d]) and more."""
    N, d = 32768, 2560
    kw = dict(K=8, D_h=80, d_model=d, dtype=eg.BF16, rows=[4449997] * 16,
              mult=np.ones((16, 3), np.uint64))
    b, p = _cfg(**kw), _cfg(flags=eg.CONV_PRENORM, **kw)
    extra = eg.engram_workspace_size(p, eg.WS_FORWARD, N) - eg.engram_workspace_size(
        b, eg.WS_FORWARD, N)
    assert extra == N * d * 4 + N * 4
    assert (eg.engram_workspace_size(p, eg.WS_BACKWARD, N)
            - eg.engram_workspace_size(b, eg.WS_BACKWARD, N)) >= N * d * 4 + N * 20


def test_invalid_configurations_rejected_before_any_launch():
    bad = [
        _cfg(K=0),
        _cfg(D_h=6),                     # 24-byte rows: not a multiple of 16 bytes
        _cfg(rows=[1009, 1009, 1008, 1009]),  # even row count
        _cfg(rows=[1009, 1009, 1, 1009]),
        _cfg(V_c=1001), _cfg(dtype=7), _cfg(flags=32),
    ]
    big = _cfg()
    big.K = 17                             # J = 34 > 32 heads
    bad.append(big)
    for c in bad:
        assert eg.engram_workspace_size(c, eg.WS_FORWARD, 64) == 0
        rc = eg.lib().engram_hash_indices(c, None, None, 1, 1, None, None, None)
        assert rc in (-1, -2), rc


def test_error_names():
    e = eg.EngramError("engram_forward", -4)
    assert "UNSUPPORTED" in str(e)
