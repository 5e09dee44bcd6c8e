"""The Python binding checks every tensor it hands to librz (dtype, rank, shape, contiguity,
device) before the library sees a pointer: the C side cannot know a buffer's element type
or length, so an unchecked tensor would be read past its end.  CPU only.  The one check a
CPU tensor cannot pass, "is on a CUDA device", is replaced here by a check without it, and
the library itself by a stub that fails the test if a call with a bad argument reaches it;
a valid call must reach it."""
import types

import pytest
import torch

import invariant_logprobs_reinforce_b200 as rz

n, d, V, R, G = 10, 64, 50, 3, 2


class ReachedLibrary(Exception):
    pass


@pytest.fixture
def cpu_rz(monkeypatch):
    def need_on_any_device(t, dtype, name, device=None):
        if not isinstance(t, torch.Tensor):
            raise TypeError(f"{name} must be a torch.Tensor")
        if t.dtype != dtype:
            raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
        if device is not None and t.device != device:
            raise ValueError(f"{name} is on {t.device}, expected {device}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        return t

    def stub():
        raise ReachedLibrary()

    monkeypatch.setattr(rz, "_need", need_on_any_device)
    monkeypatch.setattr(rz, "lib", stub)
    monkeypatch.setattr(rz, "_stream_handle", lambda stream: None)
    return rz


def _inputs():
    seg = torch.tensor([0, 3, 7, n], dtype=torch.int64)
    return dict(
        H=torch.zeros((n, d), dtype=torch.bfloat16), W_head=torch.zeros((V, d), dtype=torch.bfloat16),
        token_ids=torch.zeros(n, dtype=torch.int32), lp_rollout=torch.zeros(n), rewards=torch.zeros(R),
        seg_offsets=seg, group_ids=torch.tensor([0, 0, 1], dtype=torch.int32),
    )


def _loss_out():
    return dict(loss=torch.zeros(1), dH=torch.zeros((n, d), dtype=torch.bfloat16), dW=torch.zeros((V, d)),
                lp_out=torch.zeros(n), kappa_out=torch.zeros(n))


def _calls():
    """name -> (function, positional args builder, keyword args builder); every tensor among them is
    mutated by the tests below."""
    def loss_pos(x):
        return [x["H"], x["W_head"], x["token_ids"], x["lp_rollout"], x["rewards"], x["seg_offsets"], x["group_ids"], G]

    def seg_pos(x):
        return [torch.zeros(n), x["lp_rollout"], x["rewards"], x["seg_offsets"], x["group_ids"], G]

    events = [types.SimpleNamespace(cuda_event=0) for _ in range(8)]
    return {
        "rz_token_logprobs": (rz.rz_token_logprobs, lambda x: [x["H"], x["W_head"], x["token_ids"]],
                              lambda x: dict(lp_out=torch.zeros(n), lse_out=torch.zeros(n))),
        "rz_loss_fwd_bwd": (rz.rz_loss_fwd_bwd, loss_pos, lambda x: _loss_out()),
        "rz_loss_fwd_bwd_ex": (rz.rz_loss_fwd_bwd_ex, lambda x: loss_pos(x) + [None], lambda x: {}),
        "rz_loss_fwd_bwd_timed": (
            rz.rz_loss_fwd_bwd_timed,
            lambda x: [events] + loss_pos(x) + list(_loss_out().values()) + [torch.zeros(256, dtype=torch.uint8)],
            lambda x: {}),
        "rz_loss_fwd_bwd_streamed": (
            rz.rz_loss_fwd_bwd_streamed, lambda x: [torch.zeros((n, d), dtype=torch.bfloat16)] + loss_pos(x),
            lambda x: dict(out=dict(loss=torch.zeros(1), dH=torch.zeros((n, d), dtype=torch.bfloat16),
                                    dW=torch.zeros((V, d)), lp=torch.zeros(n), kappa=torch.zeros(n)))),
        "rz_loss_fwd_bwd_host_io": (
            rz.rz_loss_fwd_bwd_host_io, lambda x: [torch.zeros((n, d), dtype=torch.bfloat16)] + loss_pos(x),
            lambda x: dict(dH_host=torch.zeros((n, d), dtype=torch.bfloat16), dW_host=torch.zeros((V, d)),
                           out=dict(loss=torch.zeros(1), dH=torch.zeros((n, d), dtype=torch.bfloat16),
                                    dW=torch.zeros((V, d)), lp=torch.zeros(n), kappa=torch.zeros(n)))),
        "rz_segment_loss": (rz.rz_segment_loss, seg_pos,
                            lambda x: dict(loss=torch.zeros(1), kappa_out=torch.zeros(n), w_out=torch.zeros(n))),
        "rz_segment_loss_ex": (rz.rz_segment_loss_ex, lambda x: seg_pos(x) + [None], lambda x: {}),
        "rz_ratio_stats": (rz.rz_ratio_stats, lambda x: [torch.zeros(n), x["lp_rollout"], x["seg_offsets"]],
                           lambda x: dict(token_mask=torch.ones(n, dtype=torch.uint8))),
        "rz_grad_norms": (rz.rz_grad_norms, lambda x: [torch.zeros((n, d), dtype=torch.bfloat16),
                                                       torch.zeros((V, d))], lambda x: {}),
        "rz_quantize_rows_e4m3": (rz.rz_quantize_rows_e4m3, lambda x: [torch.zeros((n, d), dtype=torch.bfloat16)],
                                  lambda x: {}),
        "rz_token_logprobs_fp8": (
            rz.rz_token_logprobs_fp8,
            lambda x: [torch.zeros((n, d), dtype=torch.uint8), torch.ones(n), torch.zeros((V, d), dtype=torch.uint8),
                       torch.ones(V), x["token_ids"]],
            lambda x: dict(lp_out=torch.zeros(n), lse_out=torch.zeros(n))),
        "rz_sum_shards_f32": (rz.rz_sum_shards_f32, lambda x: [torch.zeros((4, 33))],
                              lambda x: dict(out=torch.zeros(33))),
        "rz_token_logprobs_noalloc": (rz.rz_token_logprobs_noalloc,
                                      lambda x: [x["H"], x["W_head"], x["token_ids"], torch.zeros(n)],
                                      lambda x: dict(lse_out=torch.zeros(n))),
    }


CALLS = list(_calls())
WRONG_DTYPE = {torch.float32: torch.float64, torch.bfloat16: torch.float16, torch.int32: torch.int64,
               torch.int64: torch.int32, torch.uint8: torch.int8}


def _slots(pos, kw):
    """Every tensor argument as (kind, key) with a getter and a setter on (pos, kw); the
    streamed call's `out` dict counts too."""
    slots = []
    for i, a in enumerate(pos):
        if isinstance(a, torch.Tensor):
            slots.append(("pos", i))
    for k, a in kw.items():
        if isinstance(a, torch.Tensor):
            slots.append(("kw", k))
        elif isinstance(a, dict):
            slots.extend(("out", kk) for kk, v in a.items() if isinstance(v, torch.Tensor))
    return slots


def _get(pos, kw, slot):
    kind, key = slot
    return pos[key] if kind == "pos" else (kw[key] if kind == "kw" else kw["out"][key])


def _set(pos, kw, slot, value):
    kind, key = slot
    if kind == "pos":
        pos[key] = value
    elif kind == "kw":
        kw[key] = value
    else:
        kw["out"][key] = value


def _cases():
    out = []
    for name, (_, pos_fn, kw_fn) in _calls().items():
        x = _inputs()
        for slot in _slots(pos_fn(x), kw_fn(x)):
            out.append((name, slot))
    return out


@pytest.mark.parametrize("name", CALLS)
def test_valid_arguments_reach_the_library(cpu_rz, name):
    fn, pos_fn, kw_fn = _calls()[name]
    x = _inputs()
    with pytest.raises(ReachedLibrary):
        fn(*pos_fn(x), **kw_fn(x))


@pytest.mark.parametrize("name,slot", _cases())
@pytest.mark.parametrize("mutation", ["dtype", "rank", "noncontiguous"])
def test_bad_tensor_argument_stops_before_the_library(cpu_rz, name, slot, mutation):
    fn, pos_fn, kw_fn = _calls()[name]
    x = _inputs()
    pos, kw = pos_fn(x), kw_fn(x)
    t = _get(pos, kw, slot)
    if mutation == "rank" and name == "rz_loss_fwd_bwd_timed" and slot == ("pos", len(pos) - 1):
        pytest.skip("a workspace is raw bytes: any shape of a contiguous uint8 tensor is one")
    if mutation == "dtype":
        bad, err = t.to(WRONG_DTYPE[t.dtype]), TypeError
    elif mutation == "rank":
        bad, err = (t.reshape(-1) if t.dim() == 2 else t.reshape(1, -1)), ValueError
    else:
        if t.numel() < 2:
            pytest.skip("a one-element tensor is always contiguous")
        bad = (t.t().contiguous().t() if t.dim() == 2
               else torch.zeros(2 * t.numel(), dtype=t.dtype)[::2])
        err = ValueError
        assert not bad.is_contiguous()
    _set(pos, kw, slot, bad)
    with pytest.raises(err):
        fn(*pos, **kw)


@pytest.mark.parametrize("what", ["ids", "lp_rollout", "rewards", "seg_offsets", "group_ids", "W_d", "dH", "dW"])
def test_length_mismatch_stops_before_the_library(cpu_rz, what):
    x = _inputs()
    o = _loss_out()
    longer = {"ids": ("token_ids", torch.zeros(n + 1, dtype=torch.int32)),
              "lp_rollout": ("lp_rollout", torch.zeros(n + 1)),
              "rewards": ("rewards", torch.zeros(R + 1)),
              "seg_offsets": ("seg_offsets", torch.zeros(R + 2, dtype=torch.int64)),
              "group_ids": ("group_ids", torch.zeros(R + 1, dtype=torch.int32)),
              "W_d": ("W_head", torch.zeros((V, d + 64), dtype=torch.bfloat16))}
    if what in longer:
        k, v = longer[what]
        x[k] = v
    elif what == "dH":
        o["dH"] = torch.zeros((n + 1, d), dtype=torch.bfloat16)
    else:
        o["dW"] = torch.zeros((V + 1, d))
    with pytest.raises(ValueError):
        rz.rz_loss_fwd_bwd(x["H"], x["W_head"], x["token_ids"], x["lp_rollout"], x["rewards"], x["seg_offsets"],
                           x["group_ids"], G, **o)


def test_token_mask_is_checked_against_the_call(cpu_rz):
    x = _inputs()
    lp = torch.zeros(n)
    good = rz.loss_options(clip_max=2.0, token_mask=torch.ones(n, dtype=torch.uint8))
    with pytest.raises(ReachedLibrary):
        rz.rz_segment_loss_ex(lp, x["lp_rollout"], x["rewards"], x["seg_offsets"], x["group_ids"], G, good)
    short = rz.loss_options(token_mask=torch.ones(n - 1, dtype=torch.uint8))
    with pytest.raises(ValueError):
        rz.rz_segment_loss_ex(lp, x["lp_rollout"], x["rewards"], x["seg_offsets"], x["group_ids"], G, short)
    with pytest.raises(TypeError):
        rz.loss_options(token_mask=torch.ones(n, dtype=torch.bool))
    raw = rz.rz_loss_options()
    raw.flags = rz.RZ_LOSS_TOKEN_MASK
    raw.token_mask = 4096  # a bare pointer: the binding cannot check its length
    with pytest.raises(ValueError):
        rz.rz_loss_fwd_bwd_ex(*[x[k] for k in ("H", "W_head", "token_ids", "lp_rollout", "rewards", "seg_offsets",
                                               "group_ids")], G, raw)
    with pytest.raises(TypeError):
        rz.rz_loss_fwd_bwd_ex(*[x[k] for k in ("H", "W_head", "token_ids", "lp_rollout", "rewards", "seg_offsets",
                                               "group_ids")], G, object())


def test_options_keep_the_mask_alive():
    """The struct holds only the address; the returned object also holds the tensor."""
    import gc
    m = torch.ones(7, dtype=torch.uint8)
    ptr = m.data_ptr()
    o = rz.rz_loss_options()
    o._token_mask = m
    del m
    gc.collect()
    assert o._token_mask.data_ptr() == ptr


def test_cpu_tensors_are_refused_without_a_gpu():
    """Unpatched: a tensor of the right type on the CPU is refused before the library loads."""
    x = _inputs()
    with pytest.raises(ValueError, match="CUDA"):
        rz.rz_token_logprobs(x["H"], x["W_head"], x["token_ids"])
    with pytest.raises(ValueError, match="CUDA"):
        rz.loss_options(token_mask=torch.ones(n, dtype=torch.uint8))
