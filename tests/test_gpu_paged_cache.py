"""GPU parity of the latent-cache append and the page release, through the C ABI,
against the CPU statement in oracle/paged_cache.py.

This is byte and index work, so the bar is bit-exact: the lengths, the free
count, the free stack, the block-table entries of every sequence's pages and
the cached rows every sequence can see must equal the oracle's after every
call.  A request the oracle refuses must leave all of that unchanged on the
GPU too and report the matching status.  The last test runs a few decode
steps (append the new tokens, then decode) against the decode oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import paged_cache as pc
from mla_paged_latent_decode_b200 import synth
from parity import assert_close_lse, assert_close_out, check_metadata

pytestmark = pytest.mark.gpu

PAGE = 64
STATUS = {"ok": 0, "too few free pages": 7, "free-page array full": 7}


def status_code(s):
    return STATUS.get(s, 5)  # every other refusal is a failed device check


class State:
    """The cache state twice: numpy copies for the oracle, tensors on the GPU."""

    def __init__(self, lens, pool, stride, seed, dev, capacity=None):
        g = torch.Generator().manual_seed(seed)
        kc = torch.randn((pool, PAGE, 576), generator=g).to(torch.bfloat16)
        perm = torch.randperm(pool, generator=g).to(torch.int32)
        bt = torch.zeros((len(lens), stride), dtype=torch.int32)
        cur = 0
        for i, L in enumerate(lens):
            n = pc.pages_for(L)
            bt[i, :n] = perm[cur:cur + n]
            cur += n
        cap = pool if capacity is None else capacity
        free = torch.zeros(cap, dtype=torch.int32)
        free[:pool - cur] = perm[cur:]
        self.np = dict(kc=kc.view(torch.int16).numpy().copy(), bt=bt.numpy().copy(),
                       lens=np.asarray(lens, dtype=np.int32), free=free.numpy().copy(),
                       fc=pool - cur)
        self.dev = dev
        self.kc = kc.to(dev)
        self.bt = bt.to(dev)
        self.lens = torch.tensor(lens, dtype=torch.int32, device=dev)
        self.free = free.to(dev)
        self.fc = torch.tensor([pool - cur], dtype=torch.int32, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)

    def append(self, rows):
        """rows: bf16 CPU tensor [b, s_new, 576]; returns the oracle's status string."""
        from mla_paged_latent_decode_b200 import binding
        s = self.np
        kc, bt, lens, free, fc, st = pc.append(s["kc"], s["bt"], s["lens"], s["free"], s["fc"],
                                               rows.view(torch.int16).numpy())
        self.np = dict(kc=kc, bt=bt, lens=lens, free=free, fc=fc)
        self.status.zero_()
        binding.append_latent(rows.to(self.dev), self.kc, self.bt, self.lens, self.free, self.fc,
                              self.status)
        torch.cuda.synchronize(self.dev)
        return st

    def release(self, mask):
        from mla_paged_latent_decode_b200 import binding
        s = self.np
        bt, lens, free, fc, st = pc.release(s["bt"], s["lens"], s["free"], s["fc"], mask)
        self.np = dict(kc=s["kc"], bt=bt, lens=lens, free=free, fc=fc)
        self.status.zero_()
        binding.release_pages(torch.tensor(mask, dtype=torch.int32, device=self.dev), self.bt,
                              self.lens, self.free, self.fc, self.status)
        torch.cuda.synchronize(self.dev)
        return st

    def check(self, st):
        """Bit-exact comparison of everything a reader of the cache can see."""
        s = self.np
        assert int(self.status.item()) == status_code(st), (int(self.status.item()), st)
        lens = self.lens.cpu().numpy()
        np.testing.assert_array_equal(lens, s["lens"])
        fc = int(self.fc.item())
        assert fc == s["fc"]
        free = self.free.cpu().numpy()
        np.testing.assert_array_equal(free[:fc], s["free"][:fc])
        bt = self.bt.cpu().numpy()
        kc = self.kc.view(torch.int16).cpu().numpy()
        for i, L in enumerate(s["lens"]):
            n = pc.pages_for(int(L))
            np.testing.assert_array_equal(bt[i, :n], s["bt"][i, :n])
            np.testing.assert_array_equal(pc.sequence_rows(kc, bt, lens, i),
                                          pc.sequence_rows(s["kc"], s["bt"], s["lens"], i))


def rand_rows(b, s_new, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn((b, s_new, 576), generator=g).to(torch.bfloat16)


@pytest.mark.parametrize("seed", range(3))
def test_random_appends_and_releases(cuda_device, seed):
    g = np.random.default_rng(seed)
    b = 6
    state = State([int(v) for v in g.integers(0, 200, size=b)], 48, 14, seed, cuda_device)
    for step in range(40):
        if g.random() < 0.2:
            st = state.release((g.random(b) < 0.4).astype(np.int32))
        else:
            s_new = int(g.choice([1, 2, 3, 8, 9, 63, 64, 65, 130]))
            st = state.append(rand_rows(b, s_new, 1000 * seed + step))
        state.check(st)


@pytest.mark.parametrize("L", [0, 1, 63, 64, 65, 127, 128])
@pytest.mark.parametrize("s_new", [1, 2, 7, 8, 9, 64, 65, 200])
def test_append_page_boundaries(cuda_device, L, s_new):
    state = State([L, 64 - (L % 64), 3], 24, 8, L * 1000 + s_new, cuda_device)
    st = state.append(rand_rows(3, s_new, L + s_new))
    assert st == "ok"
    state.check(st)


@pytest.mark.parametrize("b,s_new", [(1, 1), (9, 1), (600, 1), (5000, 1), (3, 300),
                                     (2, 20000), (130, 16)])
def test_append_grid_shapes(cuda_device, b, s_new):
    # batches that give one, several and many sequences per CTA, and appends
    # long enough that CTAs loop over token chunks
    g = np.random.default_rng(b + s_new)
    maxlen = 300 if b < 1000 else 16
    lens = [int(v) for v in g.integers(0, maxlen, size=b)]
    stride = pc.pages_for(maxlen + s_new)
    used = sum(pc.pages_for(v) for v in lens)
    need = sum(pc.pages_for(v + s_new) - pc.pages_for(v) for v in lens)
    state = State(lens, used + need + 5, stride, b, cuda_device)
    st = state.append(rand_rows(b, s_new, 7))
    assert st == "ok"
    state.check(st)
    assert int(state.fc.item()) == 5


@pytest.mark.parametrize("case", ["too_few_pages", "row_too_short", "negative_length",
                                  "bad_free_page", "bad_last_page", "bad_free_count"])
def test_refused_append_changes_nothing(cuda_device, case):
    state = State([100, 64, 5], 8, 6, 3, cuda_device)
    s_new = 1
    if case == "too_few_pages":
        s_new = 64 * 2     # needs 2 + 2 + 2 pages, 4 are free
    elif case == "row_too_short":
        s_new = 300        # 100 + 300 tokens need 7 pages, the row holds 6
    elif case == "negative_length":
        state.lens[2] = -1
        state.np["lens"][2] = -1
    elif case == "bad_free_page":
        state.free[state.np["fc"] - 1] = 99
        state.np["free"][state.np["fc"] - 1] = 99
    elif case == "bad_last_page":
        good = int(state.np["bt"][0, 1])
        state.bt[0, 1] = 8
        state.np["bt"][0, 1] = 8
    elif case == "bad_free_count":
        state.fc.fill_(9)  # above the stack's capacity of 8
    rows = rand_rows(3, s_new, 11)
    st = state.append(rows)
    if case == "bad_free_count":
        # the oracle has no way to hold a count above capacity: the GPU must refuse
        assert int(state.status.item()) == 5 and int(state.fc.item()) == 9
        np.testing.assert_array_equal(state.lens.cpu().numpy(), [100, 64, 5])
        return
    if case == "bad_last_page":
        # put the page back on both sides so that every visible row can be compared
        state.bt[0, 1] = good
        state.np["bt"][0, 1] = good
    assert st != "ok"
    state.check(st)


def test_refused_release_changes_nothing(cuda_device):
    state = State([100, 64, 5], 8, 3, 4, cuda_device, capacity=5)
    # 4 pages used, 4 free, capacity 5: releasing 100 + 64 tokens (3 pages) overfills
    st = state.release(np.array([1, 1, 0], dtype=np.int32))
    assert st == "free-page array full"
    state.check(st)
    st = state.release(np.array([0, 0, 1], dtype=np.int32))
    assert st == "ok"
    state.check(st)


@pytest.mark.parametrize("s_q,h_q,causal", [(1, 16, False), (1, 128, False), (2, 128, True)])
def test_decode_loop_after_appends(cuda_device, s_q, h_q, causal):
    """A few decode steps as a serving loop runs them: append this step's s_q
    new latent rows, then decode the step's queries over the grown cache."""
    from mla_paged_latent_decode_b200 import binding
    lens0 = [63, 64, 1, 200]
    b = len(lens0)
    state = State(lens0, 24, 8, 5 + h_q, cuda_device)
    for step in range(3):
        st = state.append(rand_rows(b, s_q, 50 + step))
        assert st == "ok"
        state.check(st)
        q = torch.randn((b, s_q, h_q, 576), generator=torch.Generator().manual_seed(step)).to(
            torch.bfloat16)
        md, ns = binding.get_mla_metadata(state.lens, h_q, s_q)
        out, lse = binding.mla_decode_kvcache(q.to(cuda_device), state.kc, state.bt, state.lens,
                                              512, md, ns, synth.DEFAULT_SCALE, causal)
        torch.cuda.synchronize(cuda_device)
        s = state.np
        kc = torch.from_numpy(s["kc"]).view(torch.bfloat16)
        bt = torch.from_numpy(np.maximum(s["bt"], 0))
        lens = torch.from_numpy(s["lens"])
        ref_out, ref_lse = oracle.decode(q, kc, bt, lens, synth.DEFAULT_SCALE, causal)
        assert_close_out(out.float().cpu().numpy(), ref_out, f"step {step} out")
        assert_close_lse(lse.cpu().numpy(), ref_lse, f"step {step} lse")
        inp = synth.DecodeInputs(synth.custom_workload(b, s_q, h_q, s["lens"].tolist()), 0, q,
                                 kc, bt, lens, synth.DEFAULT_SCALE, causal)
        check_metadata(inp, dict(tile_md=md.cpu(), num_splits=ns.cpu()), md.shape[0])
