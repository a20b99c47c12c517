"""Host logic of the prefill planner, through dsq_prefill_workspace_bytes (no
GPU: the planner then assumes 148 SMs, i.e. 74 CTA pairs).

The workspace holds the fp16 activations padded to whole token tiles, the
per-row shifts, and the fp32 partials when K is split; K is split only while
the pair tiles leave more than half the pairs idle, or, for the tiles of a
last wave that is at most a quarter full, when the time saved outweighs the
partials' extra pass.
"""
import pytest

Q8, Q4 = 8, 12


@pytest.fixture(scope="module")
def dsq():
    """libdsq without a device: the planner's default of 74 pairs.  With a
    CUDA device present the planner asks the device instead, so skip."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a CUDA device is present: the plan follows its SM count")
    from block_quantized_dsq_b200 import build
    build.build()
    import block_quantized_dsq_b200 as dsq
    return dsq


def _align(v, a):
    return (v + a - 1) // a * a


def test_refusals_return_zero(dsq):
    f = dsq.dsq_prefill_workspace_bytes
    assert f(7, 256, 256, 4) == 0          # unsupported type
    assert f(Q8, 256, 96, 4) == 0          # K % 256 != 0
    assert f(Q4, 0, 256, 4) == 0           # N < 1
    assert f(Q8, 256, 256, 0) == 0         # M < 1


def test_large_problem_with_a_fuller_last_wave_has_no_split(dsq):
    # 8 token tiles (256 tokens each) x 32 weight tiles = 256 pair tiles on
    # 74 pairs: 3 full waves and a last wave of 34 tiles, more than a quarter
    # of the pairs: no split, workspace = fp16 activations + shifts
    M, N, K = 2048, 8192, 4096
    assert dsq.dsq_prefill_workspace_bytes(Q8, N, K, M) == M * K * 2 + _align(M * 4, 1024)


def test_last_wave_more_than_a_quarter_full_is_not_split(dsq):
    # 128 tiles = 74 + 54
    M, N, K = 2048, 4096, 4096
    assert dsq.dsq_prefill_workspace_bytes(Q4, N, K, M) == M * K * 2 + _align(M * 4, 1024)


def test_last_wave_of_a_short_k_is_not_split(dsq):
    # 80 tiles = 74 + 6 as below, but K = 512 is two units: halving the last
    # wave saves less than the partials' extra pass costs
    M, N, K = 300, 10000, 512
    assert dsq.dsq_prefill_workspace_bytes(Q8, N, K, M) == 512 * K * 2 + _align(512 * 4, 1024)


def test_last_wave_split_ways_follow_the_idle_pairs(dsq):
    # 40 weight tiles (ragged: 10000 rows) x 2 token tiles (300 tokens) = 80
    # tiles = 74 + 6: the 6 are split 12 ways -> 2 units each -> 8 pieces
    # per tile (K = 4096: 16 units)
    M, N, K = 300, 10000, 4096
    base = 512 * K * 2 + _align(512 * 4, 1024)
    assert dsq.dsq_prefill_workspace_bytes(Q4, N, K, M) == base + 6 * 8 * 256 * 256 * 4


def test_grouped_last_wave_split(dsq):
    # 4096 + 1024 rows at 2048 tokens: 20 x 8 = 160 tiles = 2 x 74 + 12; the
    # 12 are split 6 ways (3 units each)
    M, K = 2048, 4096
    base = M * K * 2 + _align(M * 4, 1024)
    assert dsq.dsq_prefill_grouped_workspace_bytes(Q4, [4096, 1024], K, M) == base + 12 * 6 * 256 * 256 * 4


def test_small_problem_splits_k_and_holds_partials(dsq):
    # one 64-token tile x 2 weight tiles: K is split 16 ways (16 units of 256)
    M, N, K = 64, 512, 4096
    x16 = _align(M * K * 2, 1024)
    got = dsq.dsq_prefill_workspace_bytes(Q8, N, K, M)
    assert got == x16 + _align(M * 4, 1024) + 16 * M * N * 4


def test_padding_to_whole_token_tiles(dsq):
    # M = 300 -> two tiles of 256 tokens: 512 padded rows of fp16 activations
    K = 1024
    got = dsq.dsq_prefill_workspace_bytes(Q4, 8192, K, 300)
    assert got == 512 * K * 2 + _align(512 * 4, 1024)


@pytest.mark.parametrize("qtype", [Q8, Q4])
def test_workspace_grows_with_tokens_once_unsplit(dsq, qtype):
    # 64, 128, 512 and 1024 tiles: none is split (the last waves of 128, 512
    # and 1024 tiles are 54, 68 and 62 tiles, more than half of 74 pairs)
    N, K = 8192, 4096
    Ms = (512, 1024, 4096, 8192)
    sizes = [dsq.dsq_prefill_workspace_bytes(qtype, N, K, M) for M in Ms]
    assert sizes == [M * K * 2 + _align(M * 4, 1024) for M in Ms]


def test_split_partials_are_padded_to_whole_float4s(dsq):
    # one 32-token tile x 1 weight tile, K = 4096: split 16 ways; M x N = 1161
    # floats per split are padded to 1164 so every split starts float4-aligned
    M, N, K = 9, 129, 4096
    got = dsq.dsq_prefill_workspace_bytes(Q8, N, K, M)
    assert got == _align(32 * K * 2, 1024) + _align(32 * 4, 1024) + 16 * 1164 * 4


@pytest.mark.parametrize("qtype,max_m,k128", [(Q8, 1, 32768), (Q4, 1, 32768)])
def test_a_few_tokens_take_the_small_kernel(dsq, qtype, max_m, k128):
    # one token, with M x K x 4 bytes of activations <= 128 KB, runs the
    # CUDA-core kernel, which keeps its activations in shared memory: the
    # workspace is a token 256 bytes
    for M in range(1, max_m + 1):
        assert dsq.dsq_prefill_workspace_bytes(qtype, 4096, 4096, M) == 256
    assert dsq.dsq_prefill_workspace_bytes(qtype, 4096, 4096, max_m + 1) > 256
    assert dsq.dsq_prefill_workspace_bytes(qtype, 4096, k128, max_m) == 256          # exactly 128 KB
    assert dsq.dsq_prefill_workspace_bytes(qtype, 4096, k128 + 256, max_m) > 256    # just above
    assert dsq.dsq_prefill_grouped_workspace_bytes(qtype, [512, 64], 4096, max_m) == 256


@pytest.mark.parametrize("qtype,max_m", [(Q8, 1), (Q4, 1)])
def test_up_to_8_tokens_take_the_mma_sync_bridge(dsq, qtype, max_m):
    # above the CUDA-core kernel and up to 8 tokens: the rounded activations
    # [8][K] binary16 plus a 256-byte block of row shifts
    K = 4096
    for M in range(max_m + 1, 9):
        assert dsq.dsq_prefill_workspace_bytes(qtype, 1024, K, M) == 8 * K * 2 + 256
    assert dsq.dsq_prefill_workspace_bytes(qtype, 1024, K, 9) != 8 * K * 2 + 256
    # K = 16384: its activations (256 KB) do not fit; the CTA-pair plan
    assert dsq.dsq_prefill_workspace_bytes(qtype, 1024, 16384, 4) != 8 * 16384 * 2 + 256


def test_grouped_workspace_sums_the_weights_partials(dsq):
    # G = 2 weights of 512 and 128 rows at M = 64: one 64-token tile x 3
    # weight tiles, K split 16 ways (3 x 16 x 2 = 96 > 74 pairs stops the
    # doubling at 16 = the 16 units of K); each weight's partials apart
    M, K, Ns = 64, 4096, [512, 128]
    got = dsq.dsq_prefill_grouped_workspace_bytes(Q8, Ns, K, M)
    base = _align(M * K * 2, 1024) + _align(M * 4, 1024)
    assert got == base + 16 * (M * 512 + M * 128) * 4
    # a group of one is the single-weight plan
    assert dsq.dsq_prefill_grouped_workspace_bytes(Q8, [512], K, M) == dsq.dsq_prefill_workspace_bytes(Q8, 512, K, M)
