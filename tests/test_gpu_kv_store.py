"""GPU parity of the KV-store step (mla_kv_store_fp8) against the float64 oracle.

The codes and scales are integer / exact data, so the bar is bit-exact over the whole cache: the
written rows must equal the oracle's and every other byte must be left as it was (the cache is
poisoned with NaN codes and NaN scales where the step writes, and keeps its generated contents
elsewhere).  A round trip (store, then decode) is checked against the oracle decode of the
oracle-stored cache at the decode tolerances.
"""
import numpy as np
import pytest
import torch

import paged_fp8_kv_mla_b200 as M
from oracle import mla_oracle as O
from paged_fp8_kv_mla_b200 import workloads as W
from tests.oracle_io import oracle_decode

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from paged_fp8_kv_mla_b200 import build
    build.build()
    M.load()
    yield


def _latent(B, T, seed, scale_mix=True, device="cuda"):
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    x = torch.randn((B, T, 576), generator=g)
    if scale_mix:
        mags = 10.0 ** (torch.randint(-4, 4, (B, T, 1), generator=g).float())
        x = x * mags
    return x.to(torch.bfloat16).to(device)


def _poison_new_rows(inp):
    """NaN codes / NaN scales at the step's positions (the store must overwrite exactly those)."""
    blocks, scales = inp.blocks.clone(), inp.scales.clone()
    L = inp.cache_lengths.cpu().numpy().view(np.uint32).astype(np.int64)
    lut = inp.lookup_table.cpu().numpy().view(np.uint32)
    slut = None if inp.scales_lookup_table is None else inp.scales_lookup_table.cpu().numpy().view(np.uint32)
    P = blocks.shape[3]
    for b in range(len(L)):
        for i in range(inp.max_prompt_length):
            t = L[b] + i
            blk = int(lut[b, t // P])
            sblk = int(slut[b, t // P]) if slut is not None else blk
            blocks[blk, 0, inp.layer_idx, t % P, 0, :] = 0x7F
            scales[sblk, 0, inp.layer_idx, t % P, 0, 0] = float("nan")
    return blocks, scales


def _oracle_store(inp, latent, blocks, scales):
    return O.kv_store(latent.cpu().view(torch.int16).numpy().view(np.uint16),
                      inp.cache_lengths.cpu().numpy().view(np.uint32), inp.lookup_table.cpu().numpy().view(np.uint32),
                      None if inp.scales_lookup_table is None else inp.scales_lookup_table.cpu().numpy().view(np.uint32),
                      inp.layer_idx, blocks.cpu().numpy(), scales.cpu().numpy())


def _check_bitexact(blocks, scales, ref_blocks, ref_scales):
    assert np.array_equal(blocks.cpu().numpy(), ref_blocks)
    s, r = scales.cpu().numpy(), ref_scales
    assert np.array_equal(np.isnan(s), np.isnan(r))
    assert np.array_equal(s.view(np.uint32)[~np.isnan(s)], r.view(np.uint32)[~np.isnan(r)])


@pytest.mark.parametrize("cfg_i", [0, 1, 3])
def test_store_bitexact_against_oracle(cfg_i):
    inp = W.make_inputs(W.CONFIGS[cfg_i], device="cuda")
    blocks, scales = _poison_new_rows(inp)
    lat = _latent(inp.cache_lengths.shape[0], inp.max_prompt_length, 40 + cfg_i)
    ref_b, ref_s = _oracle_store(inp, lat, blocks, scales)
    M.kv_store(lat, inp.cache_lengths, inp.lookup_table, inp.scales_lookup_table, inp.layer_idx, blocks, scales)
    torch.cuda.synchronize()
    assert M.device_status() == 0
    _check_bitexact(blocks, scales, ref_b, ref_s)


def _custom(B, T, P, lengths, separate=False, seed=7, layers=1, layer_idx=0):
    cfg = W.DecodeConfig("store", batch=B, q_len=T, num_q_heads=16, page_size=P, num_layers=layers,
                         layer_idx=layer_idx, length_kind="list", length_args=tuple(lengths),
                         pool_kind="permuted", pool_factor=1.5, pool_extra=3, kv_dim=1, seed=seed,
                         separate_scales=separate, scales_pool_extra=5)
    return W.make_inputs(cfg, device="cuda")


@pytest.mark.parametrize("case", [
    dict(B=3, T=7, P=16, lengths=(0, 15, 100)),                       # page-crossing runs, first page
    dict(B=2, T=33, P=48, lengths=(5, 47), separate=True),            # page size not a power of two
    dict(B=2, T=130, P=64, lengths=(1, 64), layers=3, layer_idx=2),   # prefill-sized chunk, layer 2
])
def test_store_edge_layouts(case):
    inp = _custom(**case)
    blocks, scales = _poison_new_rows(inp)
    lat = _latent(case["B"], case["T"], 77)
    ref_b, ref_s = _oracle_store(inp, lat, blocks, scales)
    M.kv_store(lat, inp.cache_lengths, inp.lookup_table, inp.scales_lookup_table, inp.layer_idx, blocks, scales)
    torch.cuda.synchronize()
    assert M.device_status() == 0
    _check_bitexact(blocks, scales, ref_b, ref_s)


def test_store_special_rows():
    """All-zero rows (scale 1), tiny rows (subnormal codes), huge rows and single spikes."""
    inp = _custom(B=1, T=6, P=16, lengths=(10,))
    blocks, scales = _poison_new_rows(inp)
    x = torch.zeros((1, 6, 576))
    x[0, 1] = torch.linspace(-1e-30, 1e-30, 576)
    x[0, 2] = torch.randn(576) * 3e37
    x[0, 3, 17] = -5.0
    x[0, 4] = torch.randn(576)
    x[0, 4, ::7] = 0.0
    x[0, 5] = torch.randn(576) * 1e-6
    lat = x.to(torch.bfloat16).cuda()
    ref_b, ref_s = _oracle_store(inp, lat, blocks, scales)
    M.kv_store(lat, inp.cache_lengths, inp.lookup_table, inp.scales_lookup_table, inp.layer_idx, blocks, scales)
    torch.cuda.synchronize()
    assert M.device_status() == 0
    _check_bitexact(blocks, scales, ref_b, ref_s)


def test_store_rows_around_the_division_switch_and_signed_zeros():
    """Per-token scales just above and below 2^-90 (the kernel's switch between the corrected
    reciprocal product and the IEEE division), rows of negative zeros, and zeros of both signs
    inside a normal row: all bit-exact against the oracle."""
    inp = _custom(B=1, T=8, P=16, lengths=(3,))
    blocks, scales = _poison_new_rows(inp)
    g = torch.Generator().manual_seed(5)
    x = torch.randn((1, 8, 576), generator=g)
    edge = 448.0 * 2.0 ** -90
    for i, f in enumerate((1.02, 1.0, 0.98, 0.5)):
        row = x[0, i] / x[0, i].abs().max() * (edge * f)
        x[0, i] = row
    x[0, 4] = -0.0
    x[0, 5, ::3] = -0.0
    x[0, 5, 1::3] = 0.0
    x[0, 6] = torch.randn(576, generator=g) * 2.0 ** -100
    x[0, 6, 0] = 1.0                                          # tiny values beside a normal maximum
    x[0, 7] = torch.randn(576, generator=g) * 1e30
    lat = x.to(torch.bfloat16).cuda()
    ref_b, ref_s = _oracle_store(inp, lat, blocks, scales)
    M.kv_store(lat, inp.cache_lengths, inp.lookup_table, inp.scales_lookup_table, inp.layer_idx, blocks, scales)
    torch.cuda.synchronize()
    assert M.device_status() == 0
    _check_bitexact(blocks, scales, ref_b, ref_s)


def test_store_rows_where_reciprocal_and_division_differ():
    """Rows on which x * RN(1/s) and RN(x / s) round to different e4m3 codes (found by a seeded
    search): the kernel's fast path must fall back to the division exactly there."""
    rng = np.random.default_rng(16)
    x = torch.from_numpy(rng.standard_normal((4000, 576)) * 3.0).to(torch.bfloat16)
    xf = x.float().numpy()
    amax = np.abs(xf).max(1).astype(np.float32)
    s = (amax / np.float32(448)).astype(np.float32)
    inv = (np.float32(1.0) / s).astype(np.float32)

    def e4(y):
        return torch.from_numpy(np.clip(y, -448, 448).astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()

    rows = np.flatnonzero((e4(xf / s[:, None]) != e4(xf * inv[:, None])).any(1))[:16]
    assert len(rows) >= 8
    T = len(rows)
    inp = _custom(B=1, T=T, P=16, lengths=(9,))
    blocks, scales = _poison_new_rows(inp)
    lat = x[torch.from_numpy(rows)].reshape(1, T, 576).cuda()
    ref_b, ref_s = _oracle_store(inp, lat, blocks, scales)
    M.kv_store(lat, inp.cache_lengths, inp.lookup_table, inp.scales_lookup_table, inp.layer_idx, blocks, scales)
    torch.cuda.synchronize()
    assert M.device_status() == 0
    _check_bitexact(blocks, scales, ref_b, ref_s)


def test_store_then_decode_round_trip():
    inp = W.make_inputs(W.CONFIGS[3], device="cuda")
    blocks, scales = _poison_new_rows(inp)
    lat = _latent(inp.cache_lengths.shape[0], inp.max_prompt_length, 91, scale_mix=False)
    ref_b, ref_s = _oracle_store(inp, lat, blocks, scales)
    M.kv_store(lat, inp.cache_lengths, inp.lookup_table, inp.scales_lookup_table, inp.layer_idx, blocks, scales)
    out, lse = M.decode(inp.q, blocks, scales, inp.cache_lengths, inp.lookup_table, inp.scales_lookup_table,
                        inp.max_prompt_length, inp.max_cache_length, inp.layer_idx, inp.softmax_scale)
    torch.cuda.synchronize()
    assert M.device_status() == 0
    ref_inp = W.DecodeInputs(**{**inp.__dict__, "blocks": torch.from_numpy(ref_b), "scales": torch.from_numpy(ref_s)})
    rows = [0, 5, 17, 63]
    ref_out, ref_lse = oracle_decode(ref_inp, requests=rows)
    ref_out, ref_lse = ref_out[rows], ref_lse[rows]
    o = O.bf16_bits_to_f64(out.cpu().view(torch.int16).numpy().view(np.uint16))[rows]
    tol = 2e-2 * np.abs(ref_out).max() + 1e-2
    assert np.abs(o - ref_out).max() <= tol
    assert np.abs(lse.cpu().double().numpy()[rows] - ref_lse).max() <= 1e-3


def test_store_bad_page_id_is_flagged_not_written():
    inp = _custom(B=2, T=3, P=16, lengths=(3, 20))
    blocks, scales = _poison_new_rows(inp)
    lut = inp.lookup_table.clone()
    lut[1, 1] = 1 << 30                                  # request 1's new tokens land on page 1
    before = blocks.clone()
    M.kv_store(_latent(2, 3, 5), inp.cache_lengths, lut, inp.scales_lookup_table, inp.layer_idx, blocks, scales)
    torch.cuda.synchronize()
    assert M.device_status() == 6
    # request 0's three rows were written; request 1's (all on the bad page) were skipped
    changed = (blocks != before).any(dim=-1).sum().item()
    assert changed == 3
