"""A decode step with the host on both ends: lsa_copy_async (a kernel copy; either side may be
pinned host memory), lsa_append_kv / lsa_append_kv_stage_q reading q, k_new and v_new from
pinned host memory, and lsa_sparse_attn_decode writing o, lse and idx_out straight into pinned
host memory.  Every result must equal, bit for bit, the same calls on device buffers."""
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module")
def lsa(cuda_device):
    import query_aware_block_b200 as m
    return m


@pytest.mark.parametrize("nbytes", [16, 4096, 16 * 1000 + 16, 3 << 20])
def test_copy_async_between_host_and_device(lsa, nbytes):
    g = torch.Generator().manual_seed(nbytes)
    src_h = torch.randint(0, 256, (nbytes,), dtype=torch.uint8, generator=g).pin_memory()
    dst_d = torch.zeros(nbytes, dtype=torch.uint8, device=DEV)
    back_h = torch.zeros(nbytes, dtype=torch.uint8).pin_memory()
    dst2_d = torch.zeros(nbytes, dtype=torch.uint8, device=DEV)
    lsa.lsa_copy_async(dst_d, src_h)                               # host -> device
    lsa.lsa_copy_async(dst2_d, dst_d, flags=lsa.LSA_FLAG_PDL)      # device -> device, dependent
    lsa.lsa_copy_async(back_h, dst2_d, flags=lsa.LSA_FLAG_PDL)     # device -> host, dependent
    torch.cuda.synchronize()
    assert torch.equal(dst_d.cpu(), src_h)
    assert torch.equal(back_h, src_h)


def test_decode_step_with_host_inputs_and_outputs(lsa):
    case = synth.decode_case(B=2, Hkv=2, G=8, D=128, T_cap=64 * 40, seqlens=[64 * 40 - 5, 64 * 17 + 3],
                             dtype=torch.bfloat16, topk=8, n_sink=1, n_local=2, seed=611)
    B, Hq, D = case.q.shape
    Hkv, T_cap = case.k.shape[1], case.k.shape[2]
    sl = case.seqlens.to(DEV)
    last = [int(x) - 1 for x in case.seqlens.tolist()]
    k_new = torch.stack([case.k[b, :, last[b]] for b in range(B)]) * 0.5  # a new token's k, v
    v_new = torch.stack([case.v[b, :, last[b]] for b in range(B)]) * 0.5

    def run(host, staged=False, ready=False):
        k, v = case.k.to(DEV), case.v.to(DEV)
        summ = torch.zeros(B, Hkv, T_cap // 64, D, device=DEV)
        lsa.lsa_build_summaries(k, sl, summ)
        q_d = torch.empty(B, Hq, D, dtype=torch.bfloat16, device=DEV)
        if host:
            q_h, kn, vn = case.q.pin_memory(), k_new.pin_memory(), v_new.pin_memory()
            o = torch.full((B, Hq, D), 7.0, dtype=torch.bfloat16).pin_memory()
            lse = torch.full((B, Hq), 7.0).pin_memory()
            idx = torch.full((B, Hkv, 8), 99, dtype=torch.int32).pin_memory()
            if not staged:
                lsa.lsa_copy_async(q_d, q_h, flags=lsa.LSA_FLAG_PDL)
        else:
            kn, vn = k_new.to(DEV), v_new.to(DEV)
            o = torch.full((B, Hq, D), 7.0, dtype=torch.bfloat16, device=DEV)
            lse = torch.full((B, Hq), 7.0, device=DEV)
            idx = torch.full((B, Hkv, 8), 99, dtype=torch.int32, device=DEV)
            q_d.copy_(case.q.to(DEV))
        if staged:  # q, k_new, v_new in one launch (read before the wait when ready)
            f = lsa.LSA_FLAG_PDL | (lsa.LSA_FLAG_INPUTS_READY if ready else 0)
            lsa.lsa_append_kv_stage_q(q_h, q_d, kn, vn, sl, k, v, flags=f)
        else:
            lsa.lsa_append_kv(kn, vn, sl, k, v, flags=lsa.LSA_FLAG_PDL)
        lsa.lsa_sparse_attn_decode(q_d, k, v, sl, o, 8, summ=summ, n_sink=1, n_local=2,
                                   refresh_last_summary=True, idx_out=idx, lse=lse,
                                   flags=lsa.LSA_FLAG_PDL)
        torch.cuda.synchronize()
        assert lsa.lsa_device_status() == 0
        return o.cpu(), lse.cpu(), idx.cpu(), k.cpu(), v.cpu(), summ.cpu()

    dev_r = run(False)
    host_r = run(True)
    for other in (host_r, run(True, staged=True), run(True, staged=True, ready=True)):
        for a, b in zip(dev_r, other):
            assert torch.equal(a, b)
    # the appended rows are the new token's
    for b in range(B):
        assert torch.equal(host_r[3][b, :, last[b]], k_new[b])
        assert torch.equal(host_r[4][b, :, last[b]], v_new[b])


def test_stage_q_alone_copies_the_query(lsa):
    src = torch.arange(4096, dtype=torch.float32).pin_memory()
    dst = torch.zeros(4096, device=DEV)
    # B = 0: nothing appended, only the query rows copied
    st = lsa.library().lsa_append_kv_stage_q(src.data_ptr(), dst.data_ptr(), 4096 * 4, None, None,
                                             lsa.LSA_BF16, 0, 1, 64, 128, None, None, None, 0, None)
    assert st == lsa.LSA_OK
    torch.cuda.synchronize()
    assert torch.equal(dst.cpu(), src)
