"""The benchmark's roofline accounting (CPU): algorithmic bytes and FLOPs
counted element by element from the tensors each call reads and writes, and
the rule that a stale profile gives no traffic figure."""
import os
import shutil

import bench


def _nbytes(*shapes_and_sizes):
    total = 0
    for shape, size in shapes_and_sizes:
        n = 1
        for s in shape:
            n *= s
        total += n * size
    return total


def test_layer_bytes_count_every_tensor():
    B, T, H, dk, dv = 8, 4096, 16, 128, 128
    iso = _nbytes(((B, T, H, dk), 2), ((B, T, H, dk), 2), ((B, T, H, dv), 2),   # q, k, v bf16
                  ((B, T, H), 4), ((B, T, H), 4), ((B, T, H), 4),               # a, w, r
                  ((B, T, H, dv), 4),                                           # o fp32
                  ((B, H, dv, dk), 4), ((B, H), 4))                             # S_T, p_T
    assert bench.layer_bytes('iso', B, T, H, dk, dv) == iso == 685_769_216
    diag = iso + _nbytes(((B, T, H, dk), 4), ((B, H, dk), 4)) - _nbytes(((B, T, H), 4), ((B, H), 4))
    assert bench.layer_bytes('diag', B, T, H, dk, dv) == diag == 952_172_544


def test_decode_and_exact_bytes():
    B, H, d = 256, 16, 128
    dec = _nbytes(((B, H, d, d), 4), ((B, H, d, d), 4),      # S read and written
                  ((B, H, d), 4), ((B, H, d), 4),            # p read and written
                  ((B, H, d), 2), ((B, H, d), 2), ((B, H, d), 2),  # q, k, v
                  ((B, H), 4), ((B, H), 4), ((B, H, d), 4),  # a, r, w
                  ((B, H, d), 4))                            # o
    assert bench.decode_bytes(B, H, d, d) == dec
    B, T, H, dk, dv = 8, 4096, 16, 64, 64
    ex = _nbytes(((B, T, H, dk), 2), ((B, T, H, dk), 2), ((B, T, H, dv), 2),
                 ((B, T, H), 4), ((B, T, H), 4), ((B, T, H), 4), ((B, T, H, dv), 4),
                 ((B, H, dv, dk), 4), ((B, H, dk, dk), 4))
    assert bench.exact_bytes(B, T, H, dk, dv) == ex
    assert bench.exact_flops(1, 1, 1, dk, dv) == 7 * dk * dk + 7 * dv * dk


def test_backward_bytes():
    B, T, H, d = 8, 4096, 16, 128
    for variant, dim in (('iso', 1), ('diag', d)):
        wshape = (B, T, H) if variant == 'iso' else (B, T, H, d)
        inputs = _nbytes(((B, T, H, d), 2), ((B, T, H, d), 2), ((B, T, H, d), 2),
                         ((B, T, H), 4), (wshape, 4), ((B, T, H), 4))
        bwd = (2 * inputs                                   # the forward again, then the backward
               + _nbytes(((B, T, H, d), 4))                 # dO read
               + _nbytes(((B, T, H, d), 4))                 # the forward's o written
               + 2 * _nbytes(((B, H, T // 16, d, d), 4))    # state checkpoints, out and in
               + 2 * _nbytes(((B, H, T, dim), 4))           # variances, out and in
               + _nbytes(((B, T, H, d), 4), ((B, T, H, d), 4), ((B, T, H, d), 4),  # dq, dk, dv
                         ((B, T, H), 4), (wshape, 4), ((B, T, H), 4)))            # da, dw, dr
        assert bench.backward_bytes(B, T, H, d, variant) == bwd, variant


def test_kla_engine_flops():
    # per 64-token chunk and head: 52 MMAs of 128x64x16 and 8 of 128x128x16
    per = 52 * 2 * 128 * 64 * 16 + 8 * 2 * 128 * 128 * 16
    assert bench.kla_engine_flops(1, 64, 1) == per
    assert bench.kla_engine_flops(8, 4096, 16) == 8 * 16 * 64 * per
    assert bench.kla_engine_flops(1, 65, 2) == 2 * 2 * per


def test_fp32_peak_is_the_unit_count_times_the_clock():
    assert abs(bench.FP32_PEAK_TFLOPS - 148 * 128 * 2 * 1.965e9 / 1e12) < 1e-9


def test_stale_profile_gives_no_traffic(tmp_path, monkeypatch):
    """The traffic figure is scaled from the committed capture only while the
    engine's sources hash to the value recorded with it."""
    assert bench.captured_traffic(128) is not None
    per_head = bench.captured_traffic(1)
    assert bench.captured_traffic(128) == 128 * per_head
    copies = []
    for f in bench.ENGINE_SOURCES:
        dst = tmp_path / os.path.basename(f)
        shutil.copy(f, dst)
        copies.append(str(dst))
    with open(copies[0], 'a') as fh:
        fh.write('\n// changed\n')
    monkeypatch.setattr(bench, 'ENGINE_SOURCES', copies)
    assert bench.captured_traffic(128) is None
