"""The bench's algorithmic cost model (the denominators of every roofline figure).

Per (layer, channel), a block of edge U moves 4 U (3B + 2) bytes (block read, output
read-modify-write, taps or spectrum shared over the batch) and a red cell 4 (2B + 1);
the relaxed tiling has 2^(P-1-q) blocks of edge 2^q (Proposition 1 of the Flash
Inference summary, section "Kachelung-Strategie (Algorithmus 1)").  Summed, one
generation moves 4 L [(3B + 2) P / 2 + 2B + 1] bytes per (layer, channel)."""
import math

import bench


def closed_form_bytes(M, B, D, L):
    P = L.bit_length() - 1
    return M * D * 4 * L * ((3 * B + 2) * P / 2 + 2 * B + 1)


def test_headline_bytes_and_flops():
    byts, flops = bench.model_bytes_flops(18, 1, 864, 1 << 17)
    assert byts == closed_form_bytes(18, 1, 864, 1 << 17)
    assert round(byts / 1e9) == 371
    assert round(flops / 1e12, 2) == 1.56


def test_closed_form_over_shapes():
    for M, B, D, P in [(1, 1, 16, 10), (18, 4, 768, 15), (3, 2, 5, 12), (18, 8, 1024, 16)]:
        L = 1 << P
        assert bench.model_bytes_flops(M, B, D, L)[0] == closed_form_bytes(M, B, D, L)


def test_window_and_block_launches_account_for_every_byte():
    # the window launches (red cells + blocks below W) and one launch per larger block
    # size and release point together move exactly the model's bytes
    for M, B, D, P, W in [(18, 1, 864, 17, 128), (18, 4, 768, 15, 64), (2, 2, 3, 12, 32)]:
        L = 1 << P
        total = (L // W) * bench.window_bytes(M, B, D, L, W)
        for q in range(W.bit_length() - 1, P):
            total += (1 << (P - 1 - q)) * bench.level_bytes(M, B, D, L, q)
        assert total == bench.model_bytes_flops(M, B, D, L)[0]


def test_flops_take_the_cheaper_tau_per_block_size():
    # direct 2U^2 below the crossover, FFT cost above it (U = 32 and beyond)
    _, f_small = bench.model_bytes_flops(1, 1, 1, 1 << 6)
    P = 6
    want = sum((1 << (P - 1 - q)) * min(2 * 4 ** q, 10 * 2 ** q * math.log2(2 ** (q + 1)) + 6 * (2 ** q + 1) + 2 ** q)
               for q in range(P)) + 2 * (1 << P)
    assert math.isclose(f_small, want)


def test_sweep_memory_model():
    # the sweep's largest point does not fit one B200, the headline does
    assert bench.sweep_need_bytes(18, 8, 1024, 1 << 18) > 180e9
    assert bench.sweep_need_bytes(18, 1, 864, 1 << 17) < 100e9


def test_data_dependent_bytes_follow_the_oracles_schedule():
    # 20U bytes per block of the data-dependent tiling (one at powers of two, two
    # elsewhere: oracle.dd.schedule) plus 24 per red cell, per channel
    from oracle import dd
    for G, L in ((1, 16), (3, 256), (7, 1 << 12)):
        want = G * (sum(20 * U for _, _, U in dd.schedule(L)) + 24 * L)
        assert bench.dd_model_bytes(G, L) == want


def test_language_model_bytes_by_hand():
    # one layer, B = 1, D = 8, L = 4, V = 10: per token 2 (3*64 + 4*64 + 4*64 + 10*8 + 8)
    # = 1584 bytes; blocks after tokens 1, 2, 3 (U = 1, 2, 1) at 20U per chain over 8
    # chains = 640; mixer state 40 per chain and token = 1280
    assert bench.lm_model_bytes(1, 1, 8, 4, 10) == 4 * 1584 + 640 + 1280
