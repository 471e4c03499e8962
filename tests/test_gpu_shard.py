"""A shard cache on the GPU: streams b0.. and heads h0.. of larger activations, in place.

The shard's calls must give the oracle's result for its (stream, head) pairs, the same bits as an
unsharded cache fed a compact copy of those rows (same kernels, same schedule), and leave every
row of q and out outside the shard untouched."""
import pytest
import torch

from causal_video_diffusion_b200 import binding
from causal_video_diffusion_b200 import shard as S
from causal_video_diffusion_b200 import workloads as W
from tests import parity as P

pytestmark = pytest.mark.gpu


def _stream(cache, chunks, window, frames, q_canary=None):
    out = None
    for c, (q, k, v) in enumerate(chunks):
        cache.rope_kv_append(q, k, v, frames * c, frames)
        out = torch.full_like(q, float("nan")) if q_canary is None else q_canary.clone()
        cache.window_attn(q, window, out=out)
    torch.cuda.synchronize()
    assert cache.device_error() == 0
    return out


@pytest.mark.parametrize("D,split", [(64, (24, 20, 20)), (128, (44, 42, 42))])
@pytest.mark.parametrize("use_scratch", [True, False])
def test_shard_cache_in_larger_activations(D, split, use_scratch):
    act_B, act_H = 3, 5
    sh = S.Shard(b0=1, nb=2, h0=1, nh=3)
    full = W.LayerShape(B=act_B, H=act_H, D=D, Hg=12, Wg=20, d_t=split[0], d_h=split[1],
                        d_w=split[2])
    part = W.LayerShape(B=sh.nb, H=sh.nh, D=D, Hg=12, Wg=20, d_t=split[0], d_h=split[1],
                        d_w=split[2])
    cap = window = 6
    chunks = [W.gen_qkv(W.qkv_seed(41, chunk=c), full, device="cuda") for c in range(3)]
    pristine = [tuple(t.clone() for t in qkv) for qkv in chunks]
    bs, hs = slice(sh.b0, sh.b0 + sh.nb), slice(sh.h0, sh.h0 + sh.nh)

    shard_cache = binding.LayerCache(sh.nb, sh.nh, D, 12, 20, *split, cap_frames=cap,
                                     max_pos_t=9,
                                     use_scratch=use_scratch,
                                     shard=(sh.b0, sh.h0, act_B, act_H))
    got = _stream(shard_cache, chunks, window, 3)

    # every row outside the shard: q untouched by the in-place rotation, out never written
    inside = torch.zeros(act_B, 1, act_H, 1, dtype=torch.bool, device="cuda")
    inside[bs, :, hs] = True
    for (q, _, _), (q0, _, _) in zip(chunks, pristine):
        assert torch.equal(torch.where(inside, q0, q), q0)
    assert torch.isnan(got.float()[~inside.expand_as(got)]).all()
    assert not torch.isnan(got.float()[inside.expand_as(got)]).any()

    # the same rows through an unsharded cache of the shard's size: identical bits
    compact = [tuple(t[bs, :, hs].contiguous() for t in qkv) for qkv in pristine]
    oracle_in = [tuple(W.bits(t.cpu()) for t in qkv) for qkv in compact]  # before q is rotated
    ref_cache = P.make_cache(part, cap, max_pos_t=9, use_scratch=use_scratch)
    ref = _stream(ref_cache, compact, window, 3)
    assert torch.equal(got[bs, :, hs], ref)
    assert torch.equal(shard_cache.k_cache, ref_cache.k_cache)
    assert torch.equal(shard_cache.v_cache, ref_cache.v_cache)

    # and the oracle's result for those (stream, head) pairs
    ol = P.make_oracle(part, cap)
    for c, qkv in enumerate(oracle_in):
        q_rot = ol.append(*qkv, 3 * c, 3)
    want = ol.attend(q_rot, window).reshape(sh.nb, sh.nh, part.L, D).transpose(0, 2, 1, 3)
    e = P.attn_errors(P.gpu_to_f64(got[bs, :, hs]), want)
    assert e.max_abs <= P.MAX_ABS and e.mean_abs <= P.MEAN_ABS, e
    P.compare_cache(shard_cache, ol, range(sh.nh))


def test_shards_of_a_layer_fill_its_output():
    """Every shard of a 3-rank plan over one layer, each with its own cache, writes exactly its
    rows; together they give the unsharded layer's output bit for bit (one CTA per unit, so no
    unit's key range is split differently in the two runs)."""
    shape = W.LayerShape(B=2, H=4, D=128, Hg=8, Wg=16, d_t=44, d_h=42, d_w=42)
    pristine = [W.gen_qkv(W.qkv_seed(43, chunk=c), shape, device="cuda") for c in range(3)]
    whole = _stream(P.make_cache(shape, 6, max_pos_t=9, use_scratch=False),
                    [tuple(t.clone() for t in qkv) for qkv in pristine], 6, 3)
    out = torch.full_like(whole, float("nan"))
    for sh in S.plan(shape.B, shape.H, 3):
        cache = binding.LayerCache(sh.nb, sh.nh, shape.D, shape.Hg, shape.Wg, shape.d_t,
                                   shape.d_h, shape.d_w, cap_frames=6, max_pos_t=9,
                                   use_scratch=False, shard=(sh.b0, sh.h0, shape.B, shape.H))
        data = [tuple(t.clone() for t in qkv) for qkv in pristine]
        part = _stream(cache, data, 6, 3, q_canary=out)
        out = part
    assert not torch.isnan(out.float()).any()
    assert torch.equal(out, whole)


def test_shard_outside_the_activations_is_refused():
    for bad in [(0, 0, 1, 4), (1, 0, 2, 4), (0, 2, 2, 4), (-1, 0, 2, 4), (0, 0, 2, 2)]:
        b0, h0, act_B, act_H = bad
        with pytest.raises(binding.UnstepError):
            binding.LayerCache(2, 3, 64, 4, 6, 24, 20, 20, cap_frames=3, max_pos_t=3,
                               shard=(b0, h0, act_B, act_H))
