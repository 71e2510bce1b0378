"""The fp64 oracle against things other than itself (CPU only)."""
import pytest

from oracle import mla_oracle as O
from tests import oracle_checks as C


def test_brute_force_attend():
    C.check_brute_force_attend(O.attend)


@pytest.mark.parametrize("causal", [False, True])
def test_brute_force_paged(causal):
    C.check_brute_force_paged(O.decode_dense, causal)


def test_single_token():
    C.check_single_token(O.decode_dense)


def test_constant_scores():
    C.check_constant_scores(O.decode_dense)


def test_lse_is_logsumexp():
    C.check_lse_logsumexp(O.decode_dense)


def test_page_permutation_invariance():
    C.check_page_permutation(O.decode_dense)


def test_causal_rows():
    C.check_causal_row0(O.decode_dense)


def test_sparse_rules():
    C.check_sparse(O.decode_sparse, O.decode_dense)


def test_combine_reproduces_unsplit():
    C.check_combine(O.attend, O.combine)


def test_empty_key_sets():
    C.check_empty_key_sets(O.decode_dense, O.decode_sparse)


def test_e4m3_all_codes():
    C.check_e4m3(O.e4m3_to_f64)


def test_bf16_rounding():
    C.check_bf16_rounding(O.f32_round_to_bf16)


def test_fp8_record_layout():
    C.check_fp8_record(O.dequant_fp8_records)


def test_golden_two_tokens():
    C.check_golden_two_tokens(O.decode_dense)


def test_sink_brute_force():
    C.check_sink_brute_force(O.attend)


def test_sink_single_token():
    C.check_sink_single_token(O.attend)


def test_sink_as_extra_key():
    C.check_sink_as_extra_key(O.decode_dense)


def test_sink_reductions():
    C.check_sink_reductions(O.decode_dense, O.decode_sparse, O.attend, O.combine)


def test_e2m1_all_codes():
    C.check_e2m1(O.e2m1_to_f64)


def test_ue4m3_all_codes():
    C.check_ue4m3(O.ue4m3_to_f64)


def test_nvfp4_golden_row():
    C.check_nvfp4_golden(O.dequant_nvfp4)


def test_nvfp4_products_exact_in_bf16():
    C.check_nvfp4_products_exact()


def test_nvfp4_decode_brute_force():
    C.check_nvfp4_decode_brute_force(O.reference_decode)


def test_rms_norm_invariants():
    C.check_rms_norm(O.rms_norm)


def test_rope_pairs():
    C.check_rope(O.rope_rotate)


def test_q_norm_rope():
    C.check_q_norm_rope(O.q_norm_rope, O.rms_norm, O.rope_rotate)


def test_e4m3_encode():
    C.check_e4m3_encode(O.e4m3_encode, O.e4m3_to_f64)


def test_fp8_cast_rows():
    C.check_fp8_cast_rows(O.fp8_cast_rows, O.e4m3_to_f64)


def test_out_rope_fp8():
    C.check_out_rope_fp8(O.out_rope_fp8, O.fp8_cast_rows, O.rope_rotate)
