"""Synthetic layouts: segment tables tile [0, L) and follow their recipe (host only)."""
import workload


def _tiles(p):
    pos = 0
    for s, n, _m in p.segments:
        assert s == pos and n > 0
        pos += n
    return pos == p.L


def test_mixed_image_text_layout():
    p = workload.mixed_image_text()
    assert p.L == 65536 and _tiles(p)
    mods = [m for _, _, m in p.segments]
    assert all(a != b for a, b in zip(mods, mods[1:])), "images and text alternate"
    assert all(n == 576 for _, n, m in p.segments if m == workload.VIDEO)
    assert len(p.segments) > 100, "many short segments"
    assert [h.kind for h in p.heads[:4]] == ["qbound", "bound2d", "vslash", "grid"]


def test_mixed_image_text_is_seeded():
    a, b = workload.mixed_image_text(L=8192, seed=3), workload.mixed_image_text(L=8192, seed=3)
    assert a.segments == b.segments
    assert workload.mixed_image_text(L=8192, seed=4).segments != a.segments


def test_benchmark_layouts_tile_the_sequence():
    for p in (workload.qwen2_7b_video_128k(), workload.longvila_1m(), workload.qwen2_7b_video_literal(),
              workload.grid_single_head(), workload.llama3_8b_text(L=32768)):
        assert _tiles(p)
