"""GPU parity of paged decode attention against the float64 oracle.

The GPU cache is written by kvq_write and the oracle cache by the oracle; their codes
are identical (test_gpu_write), so the attention check compares against attention over
the same dequantized cache.  Tolerance: max |gpu - oracle| <= 2e-3 with float32 output;
a bfloat16 output must be that float32 result rounded to nearest even.
"""

import numpy as np
import pytest
import torch

from oracle import attention, fp
from quantized_paged_kv_02_b200 import inputs
from tests import helpers

pytestmark = pytest.mark.gpu

TOL = 2e-3
SMALL = ["c1", "c2", "c3", "c4", "c4-tok", "c4-fzp", "c4-int2", "c4-int2-tok", "c4-int2-fzp", "c5",
         "c5-fp8", "c5-bf16", "c5-int8-pc", "c5-int8-ph", "c5-int8-pt", "c5-fp8-pt"]


@pytest.fixture(scope="module", autouse=True)
def _built():
    helpers.ensure_built()


def _workload(name, **kw):
    return inputs.make(name, small=(name != "c1"), **kw)


def _decode(gc, w, out_dtype=torch.float32, lens=None, max_context=None, tables=None):
    lens = w.context_lens if lens is None else lens
    mc = int(lens.max()) if max_context is None else max_context
    tables = w.block_tables if tables is None else tables
    return gc.decode(w.q.cuda(), tables.cuda(), lens.cuda(), mc, out_dtype=out_dtype)


def _oracle(oc, w, lens=None):
    lens = w.context_lens if lens is None else lens
    return attention.decode_attention(oc, helpers.np64(w.q), w.block_tables.cpu().numpy(),
                                      lens.cpu().numpy())


@pytest.mark.parametrize("name", SMALL)
def test_decode_matches_oracle(name):
    w = _workload(name)
    static = helpers.oracle_static_scales(w)
    oc = helpers.oracle_cache(w, static)
    gc = helpers.gpu_cache(w, static=static)
    want = _oracle(oc, w)
    got = _decode(gc, w).cpu().numpy().astype(np.float64)
    err = np.abs(got - want).max()
    assert err <= TOL, err
    # bf16 output: the float32 result rounded once, so within the tolerance plus half a
    # bf16 ulp of the oracle (near zero an ulp is far below the tolerance)
    gotb = _decode(gc, w, torch.bfloat16).float().cpu().numpy().astype(np.float64)
    np.testing.assert_array_equal(gotb, fp.bf16_round(got))
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(want), 2.0 ** -126))) - 7)
    assert np.all(np.abs(gotb - want) <= TOL + ulp / 2)
    assert gc.read_fault() == (0, 0)


@pytest.mark.parametrize("name", ["c2", "c4", "c4-tok", "c4-fzp", "c4-int2", "c5-fp8"])
def test_split_count_does_not_change_result(name):
    w = _workload(name)
    static = helpers.oracle_static_scales(w)
    gc = helpers.gpu_cache(w, static=static)
    a = _decode(gc, w).cpu()
    # a larger host bound changes the split plan (more, shorter splits or fewer, longer)
    for mc in (w.max_context * 3, w.max_context * 40):
        # tables must address the larger bound: pad with block 0 (never read)
        pad = (mc + w.spec.block_size - 1) // w.spec.block_size
        tab = torch.zeros((w.spec.batch, max(pad, w.block_tables.shape[1])), dtype=torch.int32)
        tab[:, :w.block_tables.shape[1]] = w.block_tables.cpu()
        b = _decode(gc, w, max_context=mc, tables=tab).cpu()
        # only the fp32 summation order changes; the zero-point sums of the group codes
        # cancel against the products (a few bits, more with 2-bit steps)
        assert (a - b).abs().max().item() <= 3e-5


def test_edge_lengths_zero_one_and_ragged():
    w = _workload("c5")
    gc = helpers.gpu_cache(w)
    oc = helpers.oracle_cache(w)
    lens = torch.tensor([0, 1, 17], dtype=torch.int32)
    got = _decode(gc, w, lens=lens, max_context=int(w.context_lens.max())).cpu().numpy()
    want = _oracle(oc, w, lens)
    assert np.all(got[0] == 0)
    np.testing.assert_allclose(got[1:], want[1:], atol=TOL, rtol=0)
    # one token: the output is exactly the dequantized v_0 (softmax weight 1)
    K, V = oc.gather(w.block_tables.numpy()[1], 1)
    g = w.spec.num_q_heads // w.spec.num_kv_heads
    for hq in range(w.spec.num_q_heads):
        np.testing.assert_allclose(got[1, hq], V[hq // g, 0], rtol=2.0 ** -22, atol=0)


def test_block_permutation_invariance_on_gpu():
    w = _workload("c3")
    static = helpers.oracle_static_scales(w)
    gc = helpers.gpu_cache(w, static=static)
    a = _decode(gc, w).cpu()
    perm = torch.randperm(w.num_blocks, generator=torch.Generator().manual_seed(9)).to(torch.int32)
    w2 = inputs.make("c3", small=True)
    bs = w.spec.block_size
    slots = w2.slot_mapping.clone()
    slots = perm[slots.long() // bs] * bs + slots % bs
    w2.slot_mapping = slots.to(torch.int32)
    w2.block_tables = perm[w.block_tables.long()].to(torch.int32)
    gc2 = helpers.gpu_cache(w2, static=static)
    b = _decode(gc2, w2).cpu()
    assert torch.equal(a, b)


def test_bad_block_and_context_are_flagged_not_faulted():
    w = _workload("c2")
    gc = helpers.gpu_cache(w)
    tables = w.block_tables.clone()
    tables[0, 3] = w.num_blocks + 7            # out of range block id
    lens = w.context_lens.clone()
    lens[1] = 10 ** 6                          # beyond max_context
    out = gc.decode(w.q.cuda(), tables.cuda(), lens.cuda(), int(w.context_lens.max()))
    torch.cuda.synchronize()
    cnt, bits = gc.read_fault()
    assert cnt > 0 and (bits & 2) and (bits & 4)
    assert torch.all(out[1] == 0)
    assert torch.isfinite(out).all()


def test_zero_query_gives_mean_of_values():
    w = _workload("c5-fp8")
    static = helpers.oracle_static_scales(w)
    gc = helpers.gpu_cache(w, static=static)
    oc = helpers.oracle_cache(w, static)
    w.q = torch.zeros_like(w.q)
    got = _decode(gc, w).cpu().numpy()
    g = w.spec.num_q_heads // w.spec.num_kv_heads
    for b in range(w.spec.batch):
        n = int(w.context_lens[b])
        K, V = oc.gather(w.block_tables.numpy()[b], n)
        for hq in range(w.spec.num_q_heads):
            np.testing.assert_allclose(got[b, hq], V[hq // g].mean(axis=0), atol=1e-5, rtol=0)


# Length mixes for the page-balanced tensor-core schedule: (a) fewer pages than CTAs, so
# most CTAs are empty and every unit is split page by page across CTAs; (b) one long
# sequence spanning a few hundred CTAs between short and empty ones.
MIXES = {
    "sparse": [0, 1, 16, 17, 0, 33, 2, 0, 5, 48, 0, 31],
    "one-long": [4000, 3, 0, 700, 16],
}
KINDS = {
    "int8": ("int8", "per_token_head"),
    "fp8": ("fp8", "per_head"),
    "bf16": ("bf16", "none"),
    "int8-pc": ("int8", "per_channel"),
    "fp8-pc": ("fp8", "per_channel"),
    "int8-ph": ("int8", "per_head"),
    "int8-pt": ("int8", "per_tensor"),
    "fp8-pt": ("fp8", "per_tensor"),
}


@pytest.mark.parametrize("mix", sorted(MIXES))
@pytest.mark.parametrize("kind", sorted(KINDS))
def test_balanced_schedule_length_mixes(kind, mix):
    cd, mode = KINDS[kind]
    lens = MIXES[mix]
    spec = inputs.Spec("mix-%s-%s" % (kind, mix), cd, "bf16", mode, len(lens), 8, 2, 128, 16,
                       lens=lens, slack_blocks=3, seed=21)
    w = inputs.from_spec(spec)
    static = helpers.oracle_static_scales(w)
    oc = helpers.oracle_cache(w, static)
    gc = helpers.gpu_cache(w, static=static)
    got = _decode(gc, w).cpu().numpy().astype(np.float64)
    want = _oracle(oc, w)
    for b, n in enumerate(lens):
        if n == 0:
            assert np.all(got[b] == 0)
    err = np.abs(got - want).max()
    assert err <= TOL, err
    assert gc.read_fault() == (0, 0)


def test_per_channel_needs_the_tensor_core_path():
    """Per-channel scales decode on the tensor-core kernel only: head_dim 64 is refused."""
    from quantized_paged_kv_02_b200 import kvq
    spec = inputs.Spec("pc-d64", "int8", "fp16", "per_channel", 2, 8, 4, 64, 16, lens=[40, 7],
                       slack_blocks=1, seed=3)
    w = inputs.from_spec(spec)
    static = helpers.oracle_static_scales(w)
    gc = helpers.gpu_cache(w, static=static)
    oc = helpers.oracle_cache(w, static)
    helpers.assert_same_cache(gc, oc)             # the write path covers every head_dim
    with pytest.raises(kvq.KVQError):
        _decode(gc, w)


@pytest.mark.parametrize("cd", ["int4", "int2"])
@pytest.mark.parametrize("mode", ["kivi", "int4_per_token", "kivi_float_zero"])
@pytest.mark.parametrize("hq,d", [(4, 128), (16, 64)])
def test_int4_cuda_core_path(cd, mode, hq, d):
    """INT4 / INT2 caches the tensor-core kernel does not take (GQA group 2, or head_dim 64)
    run on the CUDA-core kernel, for every form."""
    spec = inputs.Spec("int4-simt", cd, "bf16", mode, 2, hq, 2, d, 64, lens=[485, 200],
                       outliers="k", slack_blocks=3, seed=5)
    w = inputs.from_spec(spec)
    oc = helpers.oracle_cache(w)
    gc = helpers.gpu_cache(w)
    helpers.assert_same_cache(gc, oc)
    got = _decode(gc, w).cpu().numpy().astype(np.float64)
    assert np.abs(got - _oracle(oc, w)).max() <= TOL
    assert gc.read_fault() == (0, 0)


@pytest.mark.parametrize("cd", ["int4", "int2"])
@pytest.mark.parametrize("mode", ["kivi", "int4_per_token", "kivi_float_zero"])
@pytest.mark.parametrize("hq", [6, 10])
def test_int4_tensor_core_path_partial_groups(cd, mode, hq):
    """GQA groups of 3 and 5 query heads on the INT4 / INT2 tensor-core kernel (N = 8 heads
    per tile, the rest masked), against the oracle."""
    spec = inputs.Spec("int4-g", cd, "bf16", mode, 2, hq, 2, 128, 64, lens=[485, 330],
                       outliers="k", slack_blocks=3, seed=9)
    w = inputs.from_spec(spec)
    oc = helpers.oracle_cache(w)
    gc = helpers.gpu_cache(w)
    got = _decode(gc, w).cpu().numpy().astype(np.float64)
    assert np.abs(got - _oracle(oc, w)).max() <= TOL
    assert gc.read_fault() == (0, 0)


@pytest.mark.parametrize("name", ["c4", "c4-int2", "c4-tok", "c5", "c3"])
def test_back_to_back_calls_share_a_workspace(name):
    """Calls enqueued back to back on one workspace, with no host synchronization between
    them, give exactly what each gives alone.  Within a call the kernels overlap (the
    low-bit block kernel runs beside the ring-split kernel, the merges start early and
    wait); a call's first kernel starts only after the previous call's last one, so no
    call reads partials another call is writing.  The second call decodes a subset of the
    batch with other queries, so its partial rows land on the first call's slots."""
    w = _workload(name)
    static = helpers.oracle_static_scales(w)
    gc = helpers.gpu_cache(w, static=static)
    B = w.spec.batch
    half = max(1, B // 2)
    q1 = w.q.cuda()
    g = torch.Generator().manual_seed(1234)
    q2 = torch.randn(w.q[:half].shape, generator=g).to(w.q.dtype).cuda()
    tab, lens = w.block_tables.cuda(), w.context_lens.cuda()
    mc = int(w.context_lens.max())
    n = max(gc.workspace_size(B, q1.shape[1], mc), gc.workspace_size(half, q1.shape[1], mc), 16)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    # each call alone, synchronized
    a1 = gc.decode(q1, tab, lens, mc, workspace=ws)
    torch.cuda.synchronize()
    a1 = a1.clone()
    a2 = gc.decode(q2, tab[:half], lens[:half], mc, workspace=ws)
    torch.cuda.synchronize()
    a2 = a2.clone()
    # the same calls enqueued back to back, three rounds
    outs = []
    for _ in range(3):
        outs.append(gc.decode(q1, tab, lens, mc, workspace=ws))
        outs.append(gc.decode(q2, tab[:half], lens[:half], mc, workspace=ws))
    torch.cuda.synchronize()
    for i, o in enumerate(outs):
        want = a1 if i % 2 == 0 else a2
        assert torch.equal(o, want), (name, i)
    assert gc.read_fault() == (0, 0)


@pytest.mark.parametrize("cd,mode", [("int4", "kivi"), ("int2", "int4_per_token"), ("int4", "kivi_float_zero")])
def test_low_bit_edge_lengths(cd, mode):
    """Low-bit caches with an empty sequence, one token, sequences held wholly in the
    residual ring (no whole 64-token group yet: 100, 191) and one just past a group (192):
    block-kernel CTAs with no blocks, ring-only splits and every split count the reduce can
    see, on the tensor-core path.  The empty sequence's output is zero."""
    spec = inputs.Spec("c4-edge", cd, "bf16", mode, 6, 16, 2, 128, 64, lens=[0, 1, 100, 191, 192, 300],
                       outliers="k", slack_blocks=2, seed=5)
    w = inputs.from_spec(spec)
    oc = helpers.oracle_cache(w)
    gc = helpers.gpu_cache(w)
    assert gc.decode_plan(spec.batch, spec.num_q_heads, w.max_context)[0] == 2   # tensor cores
    got = _decode(gc, w).cpu().numpy().astype(np.float64)
    want = _oracle(oc, w)
    assert np.all(got[0] == 0)
    assert np.abs(got - want).max() <= TOL
    assert gc.read_fault() == (0, 0)
