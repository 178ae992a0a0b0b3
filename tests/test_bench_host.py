"""Host-side logic of bench.py that needs no GPU: the code digest that decides whether a
committed ncu summary still describes the kernel source, and the summaries themselves."""
import os
import re

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_code_text_drops_comments_and_keeps_literals():
    src = ('int a = 1;  // trailing\n'
           '/* block\n   comment */ const char* s = "x//y /*z*/";\n'
           "char q = '\"'; char e = '\\\\';\n"
           '\n\n   \n'
           'asm("mov.b64 %0, {%1, %2};" : "=l"(r));  /* tail */\n')
    assert bench.code_text(src) == ('int a = 1;\n const char* s = "x//y /*z*/";\n'
                                    "char q = '\"'; char e = '\\\\';\n"
                                    'asm("mov.b64 %0, {%1, %2};" : "=l"(r));')


def test_code_digest_ignores_comments_but_not_code(tmp_path):
    a = tmp_path / 'a.cu'
    a.write_text('// header\n__global__ void k(float* p) {\n  p[0] = 1.f;  // one\n}\n')
    b = tmp_path / 'b.cu'
    b.write_text('/* another header */\n\n__global__ void k(float* p) {\n  p[0] = 1.f;\n}\n')
    c = tmp_path / 'c.cu'
    c.write_text('__global__ void k(float* p) {\n  p[0] = 2.f;\n}\n')
    assert bench.code_sha256(str(a)) == bench.code_sha256(str(b))
    assert bench.code_sha256(str(a)) != bench.code_sha256(str(c))


def test_profile_summaries_name_their_source_and_traffic():
    for kernel, (summary, source) in bench.PROFILED.items():
        text = open(os.path.join(ROOT, summary)).read()
        assert re.search(r'code_sha256:\s*[0-9a-f]{64}', text), summary
        assert re.search(r'traffic_bytes_per_launch:\s*[0-9]+', text), summary
        for src in ([source] if isinstance(source, str) else source):
            assert os.path.exists(os.path.join(ROOT, src)), src
        assert '--clock-control none' in text, summary


def test_prefill_mma_flops_by_hand():
    # T = 64 (one chunk), H = 1, d = 128, C = 64
    f = bench.prefill_mma_flops(64, 1, 128, 64)
    assert f['intra_chunk']['tf32'] == 2 * 128 * 128 * 128          # gram, M = N = K = 128
    assert f['intra_chunk']['bf16'] == 5 * 2 * 128 * 64 * 64        # W: 3 MMAs, U~: 2
    assert f['inter_chunk']['bf16'] == (2 * 128 * 128 * 128        # [W; Q~] S
                                        + 2 * 128 * 128 * 64        # K'^T U
                                        + 2 * 128 * 128 * 64)       # [0; M] U
    # a ragged tail counts as a whole chunk (the tiles are padded)
    assert bench.prefill_mma_flops(65, 2, 128, 64)['intra_chunk']['tf32'] == 4 * f['intra_chunk']['tf32']


def test_issued_mma_view_fraction():
    flops = {'intra_chunk': {'tf32': 1.1e9, 'bf16': 2.25e9}, 'inter_chunk': {'tf32': 0, 'bf16': 0}}
    r = bench.issued_mma_view(flops, {'intra_chunk': 2.0}, 2250.0)
    # bf16 2.25 GFLOP at 2.25 PFLOP/s = 1 us; tf32 1.1 GFLOP at 1.1 PFLOP/s = 1 us
    assert abs(r['intra_chunk']['ms_at_peak'] - 2e-3) < 1e-12
    assert abs(r['intra_chunk']['frac'] - 1e-3) < 1e-12
    assert 'inter_chunk' not in r


def test_dense_tile_flops_and_method_bytes_by_hand():
    # per (token, head): grams 2 C d, W and U~ 2 C d, M U C d -> 5 C d; W S, Q~ S, K'^T U -> 3 d^2
    assert bench.prefill_dense_flops(64, 1, 128, 64) == 2 * (5 * 64 * 128 + 3 * 128 * 128) * 64
    # the headline step: 47.2 GFLOP
    assert abs(bench.prefill_dense_flops(8192, 32, 128) / 1e9 - 47.24) < 0.01
    # 1,538 B per (token, head) + the final fp32 state (64 KB per head)
    assert bench.layer_method_bytes(8192, 1, 32, 128) == 8192 * 32 * 1538 + 32 * 128 * 128 * 4
    r = bench.tensor_roofline(2.25e9, 2.0, 2250.0, 1125.0)
    assert abs(r['frac'] - 5e-4) < 1e-12 and abs(r['frac_sustained'] - 1e-3) < 1e-12


def test_cosched_launch_counts_both_passes():
    # the one co-scheduled launch moves both passes' design bytes and issues both passes' MMAs
    nb = bench.prefill_bytes(8192, 32, 128)
    assert nb['prefill_cosched'] == nb['intra_chunk'] + nb['inter_chunk']
    f = bench.prefill_mma_flops(8192, 32, 128)
    for kind in ('tf32', 'bf16'):
        assert f['prefill_cosched'][kind] == f['intra_chunk'][kind] + f['inter_chunk'][kind]
    # the two-launch form's keys are still there for the separate-passes line
    assert set(nb) >= {'intra_chunk', 'inter_chunk', 'layer'}
