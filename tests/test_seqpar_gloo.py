"""Sequence parallelism across ranks (LASP+) on CPU ranks (gloo, world sizes
2 to 4): lasp_prefill's exchange -- local prefixes all-gathered in rank
order, the global prefix of the ranks before this one, the local scan seeded
with it -- reproduces the oracle's result for the whole sequences, and so
does lasp_prefill_varlen on packed batches cut at arbitrary token positions
(sequences spanning several ranks, empty sequences, empty ranks), and
lasp_prefill_backward and lasp_prefill_backward_varlen reproduce the
oracle's gradients of the whole (packed) sequences.  The device
steps are host stand-ins built from the oracle (fp64), so what is checked
here is the rank logic; the CUDA steps are checked on the GPU."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import la_inputs

D = 8  # small head dimension: the oracle takes any d


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class _HostOps:
    """The three device steps of a rank, computed by the oracle in fp64."""

    @staticmethod
    def _packed(t):
        B, n, H, d = t.shape
        return la_inputs.bits(t.reshape(B * n, H, d)), (np.arange(B + 1) * n).astype(np.int32)

    @staticmethod
    def kv_aggregate(k, v):
        import oracle
        K, cu = _HostOps._packed(k)
        V, _ = _HostOps._packed(v)
        _, st = oracle.recurrent(K, K, V, cu)  # final state from zero = sum of k_t^T v_t
        return torch.from_numpy(st)

    @staticmethod
    def state_prefix(parts, count, state_in, out=None):
        shape = parts.shape[1:] if parts is not None else (state_in if state_in is not None else out).shape
        acc = torch.zeros(shape, dtype=torch.float64) if state_in is None else state_in.clone()
        for i in range(count):
            acc += parts[i]
        if out is not None:
            out.copy_(acc)
            return out
        return acc

    @staticmethod
    def prefill(q, k, v, state_in, out_dtype):
        import oracle
        B, n, H, d = q.shape
        Q, cu = _HostOps._packed(q)
        K, _ = _HostOps._packed(k)
        V, _ = _HostOps._packed(v)
        out, _ = oracle.recurrent(Q, K, V, cu, state_in=state_in.numpy())
        return torch.from_numpy(out).reshape(B, n, H, d)

    @staticmethod
    def prefill_backward(q, k, v, dout, state_in, dstate_out, grad_dtype):
        import oracle
        B, n, H, d = q.shape
        (Q, cu), (K, _), (V, _), (G, _) = (_HostOps._packed(t) for t in (q, k, v, dout))
        dq, dk, dv, _ = oracle.backward(Q, K, V, G, cu, state_in=state_in.numpy(), dstate_out=dstate_out.numpy())
        return tuple(torch.from_numpy(x).reshape(B, n, H, d) for x in (dq, dk, dv))

    @staticmethod
    def prefill_varlen(q, k, v, cu_seqlens, max_seqlen, state_in, out_dtype):
        import oracle
        out, st = oracle.recurrent(la_inputs.bits(q), la_inputs.bits(k), la_inputs.bits(v), cu_seqlens,
                                   state_in=state_in.numpy())
        return torch.from_numpy(out), torch.from_numpy(st)

    @staticmethod
    def prefill_backward_varlen(q, k, v, dout, cu_seqlens, max_seqlen, state_in, dstate_out, grad_dtype):
        import oracle
        res = oracle.backward(*(la_inputs.bits(t) for t in (q, k, v, dout)), np.asarray(cu_seqlens, np.int32),
                              state_in=state_in.numpy(), dstate_out=dstate_out.numpy())
        return tuple(torch.from_numpy(x) for x in res)


def _worker(rank, world, port, lens, result_path):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        from linear_attention_blocked_b200 import seqpar
        B, H = 2, 3
        N = sum(lens)
        q, k, v = la_inputs.qkv((B, N, H, D), seed=61, scale=0.5)
        sin = torch.from_numpy(np.random.default_rng(62).standard_normal((B, H, D, D)) * 0.3)
        a = sum(lens[:rank])
        part = lambda t: t[:, a:a + lens[rank]].contiguous()
        out, final = seqpar.lasp_prefill(part(q), part(k), part(v), state_in=sin, ops=_HostOps)
        shares = [None] * world
        dist.all_gather_object(shares, (out.numpy(), final.numpy()))
        if rank == 0:
            Q, cu = _HostOps._packed(q)
            K, _ = _HostOps._packed(k)
            V, _ = _HostOps._packed(v)
            ref, rst = oracle.recurrent(Q, K, V, cu, state_in=sin.numpy())
            ref = ref.reshape(B, N, H, D)
            got = np.concatenate([o for o, _ in shares], axis=1)
            scale = np.abs(ref).max()
            ok = got.shape == ref.shape and np.abs(got - ref).max() <= 1e-10 * scale
            for _, f in shares:
                ok &= np.abs(f - rst).max() <= 1e-10 * np.abs(rst).max()
            with open(result_path, "w") as fh:
                fh.write("ok" if ok else f"mismatch {np.abs(got - ref).max()}")
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("lens", [[40, 77], [130, 1, 59]])
def test_ranks_reproduce_the_whole_sequence(tmp_path, oracle_mod, lens):
    result = tmp_path / "result.txt"
    mp.start_processes(_worker, args=(len(lens), _free_port(), lens, str(result)), nprocs=len(lens), join=True,
                       start_method="spawn")
    assert result.read_text() == "ok"


def _varlen_worker(rank, world, port, lens, bounds, result_path):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        from linear_attention_blocked_b200 import seqpar
        H = 2
        cu = la_inputs.cu_seqlens_from_lengths(lens)
        T = int(cu[-1])
        q, k, v = la_inputs.qkv((T, H, D), seed=63, scale=0.5)
        sin = torch.from_numpy(np.random.default_rng(64).standard_normal((len(lens), H, D, D)) * 0.3)
        a, b = int(bounds[rank]), int(bounds[rank + 1])
        out, st, plan = seqpar.lasp_prefill_varlen(q[a:b].contiguous(), k[a:b].contiguous(), v[a:b].contiguous(),
                                                   cu, bounds, state_in=sin, ops=_HostOps)
        shares = [None] * world
        dist.all_gather_object(shares, (out.double().numpy(), st.double().numpy(), plan.seq0, plan.ends_here))
        if rank == 0:
            ref, rst = oracle.recurrent(la_inputs.bits(q), la_inputs.bits(k), la_inputs.bits(v), cu,
                                        state_in=sin.numpy())
            got = np.concatenate([o for o, _, _, _ in shares], axis=0)
            ok = got.shape == ref.shape and np.abs(got - ref).max() <= 1e-10 * np.abs(ref).max()
            final = np.full(rst.shape, np.nan)
            seen = np.zeros(len(lens), int)
            for _, s_, seq0, ends in shares:
                for i in np.nonzero(ends)[0]:
                    final[seq0 + i] = s_[i]
                    seen[seq0 + i] += 1
            ok &= bool(np.all(seen == 1))
            ok &= bool(np.abs(final - rst).max() <= 1e-10 * np.abs(rst).max())
            with open(result_path, "w") as fh:
                fh.write("ok" if ok else f"mismatch seen={seen.tolist()}")
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("lens,bounds", [
    ([50, 0, 130, 7, 0, 200, 1], None),                 # cut evenly into 3 ranks
    ([20, 400, 30], None),                              # the long sequence spans all 4 ranks
    ([50, 0, 130, 7, 0, 200, 1], [0, 50, 50, 300, 388]),  # cuts on sequence edges, an empty rank
    ([3, 0, 0], [0, 3, 3]),                             # trailing empty sequences on the last rank
])
def test_varlen_ranks_reproduce_the_packed_batch(tmp_path, oracle_mod, lens, bounds):
    from linear_attention_blocked_b200 import seqpar
    T = sum(lens)
    world = 4 if bounds is None and len(lens) == 3 else (3 if bounds is None else len(bounds) - 1)
    bounds = np.asarray(bounds if bounds is not None else seqpar.split_tokens(T, world))
    result = tmp_path / "result.txt"
    mp.start_processes(_varlen_worker, args=(world, _free_port(), lens, bounds, str(result)), nprocs=world,
                       join=True, start_method="spawn")
    assert result.read_text() == "ok"


def _backward_worker(rank, world, port, lens, result_path):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        from linear_attention_blocked_b200 import seqpar
        B, H = 2, 2
        N = sum(lens)
        q, k, v = la_inputs.qkv((B, N, H, D), seed=71, scale=0.5)
        g, _, _ = la_inputs.qkv((B, N, H, D), seed=72, scale=0.5)
        rng = np.random.default_rng(73)
        sin = torch.from_numpy(rng.standard_normal((B, H, D, D)) * 0.3)
        gs = torch.from_numpy(rng.standard_normal((B, H, D, D)) * 0.3)
        a = sum(lens[:rank])
        part = lambda t: t[:, a:a + lens[rank]].contiguous()  # noqa: E731
        dq, dk, dv, dsin = seqpar.lasp_prefill_backward(part(q), part(k), part(v), part(g), state_in=sin,
                                                        dstate_out=gs, ops=_HostOps)
        shares = [None] * world
        dist.all_gather_object(shares, tuple(x.numpy() for x in (dq, dk, dv, dsin)))
        if rank == 0:
            (Q, cu), (K, _), (V, _), (G, _) = (_HostOps._packed(t) for t in (q, k, v, g))
            ref = oracle.backward(Q, K, V, G, cu, state_in=sin.numpy(), dstate_out=gs.numpy())
            ok = True
            for i in range(3):
                got = np.concatenate([sh[i] for sh in shares], axis=1).reshape(B * N, H, D)
                ok &= bool(np.abs(got - ref[i]).max() <= 1e-10 * np.abs(ref[i]).max())
            for sh in shares:
                ok &= bool(np.abs(sh[3] - ref[3]).max() <= 1e-10 * np.abs(ref[3]).max())
            with open(result_path, "w") as fh:
                fh.write("ok" if ok else "mismatch")
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("lens", [[40, 77], [130, 1, 59]])
def test_backward_ranks_reproduce_the_whole_sequence(tmp_path, oracle_mod, lens):
    result = tmp_path / "result.txt"
    mp.start_processes(_backward_worker, args=(len(lens), _free_port(), lens, str(result)), nprocs=len(lens),
                       join=True, start_method="spawn")
    assert result.read_text() == "ok"


def _varlen_backward_worker(rank, world, port, lens, bounds, result_path):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        from linear_attention_blocked_b200 import seqpar
        H = 2
        cu = la_inputs.cu_seqlens_from_lengths(lens)
        T = int(cu[-1])
        q, k, v = la_inputs.qkv((T, H, D), seed=81, scale=0.5)
        g, _, _ = la_inputs.qkv((T, H, D), seed=82, scale=0.5)
        rng = np.random.default_rng(83)
        sin = torch.from_numpy(rng.standard_normal((len(lens), H, D, D)) * 0.3)
        gs = torch.from_numpy(rng.standard_normal((len(lens), H, D, D)) * 0.3)
        a, b = int(bounds[rank]), int(bounds[rank + 1])
        part = lambda t: t[a:b].contiguous()  # noqa: E731
        dq, dk, dv, dsin, plan = seqpar.lasp_prefill_backward_varlen(part(q), part(k), part(v), part(g), cu, bounds,
                                                                     state_in=sin, dstate_out=gs, ops=_HostOps)
        shares = [None] * world
        dist.all_gather_object(shares, (tuple(x.double().numpy() for x in (dq, dk, dv, dsin)), plan.seq0,
                                        plan.starts_here))
        if rank == 0:
            ref = oracle.backward(*(la_inputs.bits(t) for t in (q, k, v, g)), cu, state_in=sin.numpy(),
                                  dstate_out=gs.numpy())
            ok = True
            for i in range(3):
                got = np.concatenate([sh[0][i] for sh in shares], axis=0)
                ok &= got.shape == ref[i].shape and bool(np.abs(got - ref[i]).max() <= 1e-10 * np.abs(ref[i]).max())
            dsin_all = np.full(ref[3].shape, np.nan)
            seen = np.zeros(len(lens), int)
            for (grads, seq0, starts) in shares:
                for j in np.nonzero(starts)[0]:
                    dsin_all[seq0 + j] = grads[3][j]
                    seen[seq0 + j] += 1
            ok &= bool(np.all(seen == 1))
            ok &= bool(np.abs(dsin_all - ref[3]).max() <= 1e-10 * np.abs(ref[3]).max())
            with open(result_path, "w") as fh:
                fh.write("ok" if ok else f"mismatch seen={seen.tolist()}")
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("lens,bounds", [
    ([50, 0, 130, 7, 0, 200, 1], None),                 # cut evenly into 3 ranks
    ([20, 400, 30], None),                              # the long sequence spans all 4 ranks
    ([50, 0, 130, 7, 0, 200, 1], [0, 50, 50, 300, 388]),  # cuts on sequence edges, an empty rank
    ([3, 0, 0], [0, 3, 3]),                             # trailing empty sequences on the last rank
])
def test_varlen_backward_ranks_reproduce_the_packed_batch(tmp_path, oracle_mod, lens, bounds):
    """lasp_prefill_backward_varlen: every rank's gradients of its tokens, and
    each sequence's dS_in from the rank where it starts, equal the oracle's
    gradients of the whole packed batch."""
    from linear_attention_blocked_b200 import seqpar
    T = sum(lens)
    world = 4 if bounds is None and len(lens) == 3 else (3 if bounds is None else len(bounds) - 1)
    bounds = np.asarray(bounds if bounds is not None else seqpar.split_tokens(T, world))
    result = tmp_path / "result.txt"
    mp.start_processes(_varlen_backward_worker, args=(world, _free_port(), lens, bounds, str(result)),
                       nprocs=world, join=True, start_method="spawn")
    assert result.read_text() == "ok"

