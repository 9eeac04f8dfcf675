"""Host-side checks of the tiled cache layout exposed by the Python binding (no GPU).

The layout is the one include/qjl.h documents: per (sequence, kv head) a slab of
cap/64 tiles, each holding its 64 tokens' sign words, outlier sign words, norms,
value codes and (scale, zero) pairs, section after section.
"""

import numpy as np
import pytest

torch = pytest.importorskip("torch")

from decode_attention_qjl_b200 import qjl as Q  # noqa: E402


@pytest.mark.parametrize("m,m_out", [(256, 64), (128, 0), (512, 32)])
def test_sections_address_the_documented_bytes(m, m_out):
    B, Hkv, cap = 2, 3, 130  # rounds up to 192 slots = 3 tiles
    c = Q.QJLCache.allocate(B, Hkv, cap, m, m_out, 8, device="cpu")
    assert c.cap == 192 and c.tiles.shape == (B, Hkv, 3, Q.tile_bytes(m, m_out))
    # fill every byte with a function of its position, then read it back through the views
    flat = torch.arange(c.tiles.numel(), dtype=torch.int64)
    c.tiles.copy_((flat * 2654435761 % 251).to(torch.uint8).view_as(c.tiles))
    raw = c.tiles.numpy()
    tb = Q.tile_bytes(m, m_out)
    rng = np.random.default_rng(0)
    for _ in range(50):
        b, h, t = int(rng.integers(B)), int(rng.integers(Hkv)), int(rng.integers(c.cap))
        tile = raw[b, h, t // 64]
        j = t % 64
        off = 0
        for name, nb in (("kbits", m // 8), ("kbits_out", m_out // 8), ("knorm", 4), ("vcode", 64), ("vsz", 16)):
            want = tile[off + j * nb: off + (j + 1) * nb]
            if name == "vcode":  # group g of token j sits at 16-byte chunk g ^ ((j >> 1) & 3)
                want = np.concatenate([want[16 * (g ^ ((j >> 1) & 3)):][:16] for g in range(4)])
            got = c.section(name)[b, h, t].numpy().reshape(-1).view(np.uint8)
            assert np.array_equal(got, want), (name, b, h, t)
            off += 64 * nb
        assert off == tb
    assert c.section("kbits").shape == (B, Hkv, c.cap, m // 32)
    assert c.section("kbits_out").shape == (B, Hkv, c.cap, m_out // 32)
    assert c.section("vsz").shape == (B, Hkv, c.cap, 4, 2)
