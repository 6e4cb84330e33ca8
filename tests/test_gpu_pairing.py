"""GPU: the tile-pairing schedule that bsa_pair_tiles writes for the paired
attention (a scheduling step of this implementation; the pages have no
counterpart).  The schedule must be a valid reordering of the selection's
lists, whatever pairs the heuristic picks:

* every video query block of every (b, h) appears in exactly one entry, the
  text query blocks in the leading text entries;
* each tile's reordered list is a permutation of its own list;
* a pair's two lists start with the same c blocks: exactly the video blocks
  both lists hold (ascending), then every text block; the rest of each list
  is ascending;
* on the full HunyuanVideo lists the matched pairs share at least half of
  their video blocks (a regression guard for the matching heuristic).

The workspace is read with the layout the library carves it into: the
pairing scratch (list bit sets, then 8 candidate partners per block as
uint16), the schedule [B*Hd, pairs, 4] int32 and the lists
[B*Hd, pairs, 2, kmax] int32, each part 256-byte aligned.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_permute_b200 as bsa
import synthetic
from parity import custom_workload

pytestmark = pytest.mark.gpu

CAND = 8   # candidate partners per query block kept in the pairing scratch


def _r256(x):
    return (x + 255) // 256 * 256


def read_schedule(plan, ws, kmax):
    info = plan.info
    nb, nb_text = info.nb, info.nb_text
    bh = info.batch * info.heads
    nbw = (nb + 31) // 32
    text_pairs = (nb_text + 1) // 2
    pph = text_pairs + (nb + 1) // 2
    scratch = bh * nb * nbw * 4 + 256 + bh * nb * CAND * 2
    off_sched = _r256(scratch)
    off_lists = off_sched + _r256(bh * pph * 4 * 4)
    raw = ws.cpu().numpy()
    sched = raw[off_sched:off_sched + bh * pph * 16].view(np.int32).reshape(bh, pph, 4)
    lists = raw[off_lists:off_lists + bh * pph * 2 * kmax * 4].view(np.int32).reshape(bh, pph, 2, kmax)
    return sched, lists, text_pairs


def check_schedule(plan, idx, cnt, ws):
    """Validity of the schedule; returns (shared video blocks counted once per
    tile, video blocks in all lists) over the matched pairs."""
    kmax = idx.shape[-1]
    nb, nb_text = plan.info.nb, plan.info.nb_text
    sched, lists, tp = read_schedule(plan, ws, kmax)
    idx_np = idx.cpu().numpy().reshape(-1, nb, kmax)
    cnt_np = cnt.cpu().numpy().reshape(-1, nb)
    text = np.arange(nb, nb + nb_text)
    shared_total, video_total = 0, 0
    for bh in range(sched.shape[0]):
        for t in range(tp):
            i0, i1, c = sched[bh, t, :3]
            assert i0 == nb + 2 * t
            assert i1 == (nb + 2 * t + 1 if 2 * t + 1 < nb_text else -1)
            assert c == (nb + nb_text if i1 >= 0 else 0)
        tiles = []
        for e in range(tp, sched.shape[1]):
            i, j, c = (int(x) for x in sched[bh, e, :3])
            assert i >= 0, f"empty video entry {e} of head {bh}"
            tiles.append(i)
            li_orig = idx_np[bh, i, :cnt_np[bh, i]]
            li = lists[bh, e, 0, :cnt_np[bh, i]]
            assert np.array_equal(np.sort(li), np.sort(li_orig))
            if j < 0:
                assert c == 0 and np.array_equal(li, li_orig)
                continue
            tiles.append(j)
            lj_orig = idx_np[bh, j, :cnt_np[bh, j]]
            lj = lists[bh, e, 1, :cnt_np[bh, j]]
            assert np.array_equal(np.sort(lj), np.sort(lj_orig))
            both = np.intersect1d(li_orig[li_orig < nb], lj_orig[lj_orig < nb])
            ns = len(both)
            assert c == ns + nb_text
            assert np.array_equal(li[:ns], both) and np.array_equal(lj[:ns], both)
            assert np.array_equal(li[ns:c], text) and np.array_equal(lj[ns:c], text)
            for rest in (li[c:], lj[c:]):
                assert np.all(np.diff(rest) > 0)
            shared_total += 2 * ns
            video_total += int((li_orig < nb).sum() + (lj_orig < nb).sum())
        assert np.array_equal(np.sort(tiles), np.arange(nb)), f"head {bh}: tiles not a partition"
    return shared_total, video_total


CASES = {
    "hy_ragged_text": custom_workload("hy_ragged_text", 1, 6, 12, 20, 1, 8, 16, 3, 128, 130,
                                      "bf16", 0, 0.3),
    "wan_d64_b2": custom_workload("wan_d64_b2", 2, 9, 10, 20, 4, 4, 8, 2, 64, 0, "bf16", 0, 0.25),
    "wan_topp": custom_workload("wan_topp", 1, 9, 10, 20, 4, 4, 8, 3, 128, 0, "bf16", 1, 0.9),
    "odd_text": custom_workload("odd_text", 2, 5, 9, 20, 1, 8, 16, 2, 128, 300, "bf16", 0, 0.4),
    # 224 blocks: the candidate window (79 blocks each side) is narrower than a head
    "window_lt_nb": custom_workload("window_lt_nb", 1, 16, 32, 56, 4, 4, 8, 2, 128, 0, "bf16", 0,
                                    0.1),
    "single_token": custom_workload("single_token", 1, 1, 1, 1, 1, 8, 16, 1, 128, 0, "bf16", 0, 1.0),
}


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    bsa.load()
    return torch.device("cuda", 0)


def _pair(w, dev):
    q, k, _ = synthetic.make_qkv(w)
    qd, kd = q.to(dev), k.to(dev)
    plan = bsa.plan_for(w, dev)
    qc, kc = plan.centroids(qd, kd)
    idx, cnt = plan.select_centroids(qc, kc, w.mode, w.params)
    ws = plan.pair_tiles(idx, cnt)
    plan.check_status()
    return plan, idx, cnt, ws


@pytest.mark.parametrize("name", list(CASES))
def test_pair_schedule_is_valid(name, dev):
    plan, idx, cnt, ws = _pair(CASES[name], dev)
    check_schedule(plan, idx, cnt, ws)


def test_pair_schedule_full_hunyuan(dev):
    """The full HunyuanVideo workload as bsa_forward pairs it."""
    plan, idx, cnt, ws = _pair(synthetic.workload("hunyuan"), dev)
    shared, video = check_schedule(plan, idx, cnt, ws)
    frac = shared / video
    print(f"hunyuan: matched pairs share {frac:.3f} of their video blocks")
    assert frac >= 0.5


@pytest.mark.parametrize("name", ["hy_ragged_text", "wan_d64_b2", "wan_topp", "window_lt_nb"])
def test_forward_pairing_equals_pair_tiles(name, dev):
    """bsa_forward hands the pairing the bit sets the selection writes beside
    its lists (no separate bit-set pass): the bit sets, the schedule and the
    reordered lists in the forward's workspace equal those bsa_pair_tiles
    derives from the same lists, bit for bit."""
    w = CASES[name]
    q, k, v = synthetic.make_qkv(w)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    plan = bsa.plan_for(w, dev)
    kmax = plan.kmax_for(w.mode, w.params)
    ws = torch.zeros(plan.workspace_size(kmax)[1], dtype=torch.uint8, device=dev)
    _, idx, cnt = plan.forward(qd, kd, vd, w.mode, w.params, kmax=kmax, workspace=ws,
                               return_lists=True)
    ref = plan.pair_tiles(idx, cnt)
    plan.check_status()
    info = plan.info
    bh, nb = info.batch * info.heads, info.nb
    # the forward's workspace: Q and K centroids, its own lists and counts, then
    # the pairing workspace
    off = 2 * _r256(bh * nb * info.head_dim * 4) + _r256(bh * nb * kmax * 4) + _r256(bh * nb * 4)
    fwd = ws[off:]
    nbits = bh * nb * ((nb + 31) // 32) * 4
    assert torch.equal(fwd[:nbits].cpu(), ref[:nbits].cpu())
    sched_f, lists_f, tp = read_schedule(plan, fwd, kmax)
    sched_r, lists_r, _ = read_schedule(plan, ref, kmax)
    assert np.array_equal(sched_f, sched_r)
    cnt_np = cnt.cpu().numpy().reshape(bh, nb)
    for b in range(bh):
        for e in range(tp, sched_r.shape[1]):
            for x in range(2):
                t = int(sched_r[b, e, x])
                if t >= 0:
                    n = cnt_np[b, t]
                    assert np.array_equal(lists_f[b, e, x, :n], lists_r[b, e, x, :n]), (b, e, x)
    check_schedule(plan, idx, cnt, fwd)
