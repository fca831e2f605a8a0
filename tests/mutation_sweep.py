"""Mutation sweep over the CPU oracle: plants one plausible slip at a time in
a temporary copy of `oracle/` and runs the pin suites (test_oracle_pins.py,
test_oracle_boot_pins.py) against that copy.  A pin set that is independent
of the oracle must fail on every slip; a slip that passes every pin would
mark a step left unpinned.

Each entry is (what the slip is, file, text, replacement, which occurrence,
the pin expected to catch it).  The replacement is applied to the copy only;
the repository's oracle is never touched.

    python tests/mutation_sweep.py            # every slip, full pin suite each
    python tests/mutation_sweep.py 0 15 21    # chosen slips
    python tests/mutation_sweep.py --targeted # run only each slip's own pin
    python tests/mutation_sweep.py --jobs 4   # four slips at a time, threads split between them
"""
import os
import shutil
import subprocess
import sys
import tempfile

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PINS = [os.path.join(ROOT, "tests", f) for f in ("test_oracle_pins.py", "test_oracle_boot_pins.py")]
C = "ckks_oracle.c"

MUTATIONS = [
    ("NTT twiddle index", C,
     "u64 w = t->fw[m + i];", "u64 w = t->fw[i + 1];", 0,
     "test_ntt_of_monomials_is_the_evaluation_vector"),
    ("INTT without n^-1", C,
     "a[j] = mulmod(a[j], t->n_inv, q);", "a[j] = a[j] % q;", 0,
     "test_ntt_roundtrip_identity"),
    ("psi: largest root instead of smallest", C,
     "if (cur < best) best = cur;", "if (cur > best) best = cur;", 0,
     "test_psi_is_smallest_primitive_root"),
    ("prime scan steps by 4n", C,
     "        c -= m;\n    }", "        c -= 2 * m;\n    }", 0,
     "test_primes_follow_the_scan_rule"),
    ("Miller-Rabin squaring loop one short", C,
     "for (int r = 1; r < s; ++r) {", "for (int r = 2; r < s; ++r) {", 0,
     "test_primes_follow_the_scan_rule"),
    ("NTT-domain automorphism without bit reversal", C,
     "return (int)bitrev((e - 1) / 2, lg);", "return (int)((e - 1) / 2);", 0,
     "test_automorph_ntt_permutation_matches_coefficients"),
    ("coefficient automorphism drops the X^n = -1 sign", C,
     "else out[e - n] = submod(out[e - n], in[j], q);",
     "else out[e - n] = addmod(out[e - n], in[j], q);", 0,
     "test_automorph_coeff_monomials"),
    ("basis conversion skips the q-hat inverse", C,
     "mulmod(x[(size_t)i * n + k], hat_inv[i], src[i])", "(x[(size_t)i * n + k] % src[i])", 0,
     "test_basis_conversion_crt_identity"),
    ("basis conversion: q-hat reduced by the wrong prime", C,
     "pt = mulmod(pt, src[i2] % dst[t], dst[t]);", "pt = mulmod(pt, src[i2] % src[i], dst[t]);", 0,
     "test_basis_conversion_crt_identity"),
    ("ModUp leaves the digit's own limbs empty", C,
     "for (int t = lo; t < hi; ++t)\n            memcpy(dj",
     "for (int t = lo; t < lo; ++t)\n            memcpy(dj", 0,
     "test_modup_crt_identity"),
    ("ModUp converts NTT values (no INTT)", C,
     "for (int l = 0; l < L; ++l) ntt_inv_one(coef", "for (int l = 0; l < 0; ++l) ntt_inv_one(coef", 0,
     "test_modup_crt_identity"),
    ("ModUp output left in the coefficient domain", C,
     "ntt_fwd_one(row, &tabs[dst_idx[c]], n);", "(void)row;", 0,
     "test_modup_crt_identity"),
    ("key inner product: key halves swapped", C,
     "key[(((size_t)j * 2 + c) * LK + t) * n + k];",
     "key[(((size_t)j * 2 + (1 - c)) * LK + t) * n + k];", 0,
     "test_rotation_decrypts_to_slot_rotation_config1"),
    ("key inner product without the automorphism", C,
     "digits[((size_t)j * LK + t) * n + src[k]];", "digits[((size_t)j * LK + t) * n + k];", 0,
     "test_rotation_decrypts_to_slot_rotation_config1"),
    ("key inner product drops the last digit", C,
     "for (int j = 0; j < dnum; ++j) {\n                    u64 d",
     "for (int j = 0; j + 1 < dnum; ++j) {\n                    u64 d", 0,
     "test_rotation_decrypts_to_slot_rotation_config1"),
    ("ModDown without P^-1", C,
     "mulmod(submod(a[(size_t)i * n + k], ci[k], mods[i]), pinv[i], mods[i]);",
     "submod(a[(size_t)i * n + k], ci[k], mods[i]);", 0,
     "test_moddown_floor_identity"),
    ("ModDown adds the conversion", C,
     "mulmod(submod(a[(size_t)i * n + k], ci[k], mods[i]), pinv[i], mods[i]);",
     "mulmod(addmod(a[(size_t)i * n + k], ci[k], mods[i]), pinv[i], mods[i]);", 0,
     "test_moddown_floor_identity"),
    ("ModDown subtracts coefficients from NTT values", C,
     "ntt_fwd_one(ci, &tabs[i], n);", "(void)ci;", 0,
     "test_moddown_floor_identity"),
    ("hoisted rotation adds c0 unrotated", C,
     "o[at] = addmod(rot0[at], ks[at], mods[i]);", "o[at] = addmod(c0[at], ks[at], mods[i]);", 0,
     "test_rotation_decrypts_to_slot_rotation_config1"),
    ("unhoisted rotation adds c0 unrotated", C,
     "o[at] = addmod(rot0[at], ks[at], mods[i]);", "o[at] = addmod(c0[at], ks[at], mods[i]);", 1,
     "test_unhoisted_rotation_order_decrypts_and_differs_in_low_bits"),
    ("unhoisted rotation applies the automorphism twice", C,
     "inner_one(dig, keys[r], 1, acc", "inner_one(dig, keys[r], galois[r], acc", 0,
     "test_unhoisted_rotation_order_decrypts_and_differs_in_low_bits"),
    ("rescale by the wrong prime's inverse on limb 0", C,
     "u64 inv = invmod(mods[l] % qi, qi);",
     "u64 inv = invmod(mods[l] % qi, qi); inv = i ? inv : invmod(mods[l - 1] % qi, qi);", 0,
     "test_rescale_is_exact_floor"),
    ("rescale subtracts the wrong way", C,
     "row[k] = mulmod(submod(in[(size_t)i * n + k], row[k], qi), inv, qi);",
     "row[k] = mulmod(submod(row[k], in[(size_t)i * n + k], qi), inv, qi);", 0,
     "test_rescale_is_exact_floor"),
    ("tensor product drops a cross term", C,
     "addmod(mulmod(a0[at], b1[at], q), mulmod(a1[at], b0[at], q), q);",
     "mulmod(a0[at], b1[at], q);", 0,
     "test_rotation_and_relin_config3_params"),
    ("tensor product: d2 from a transposed operand", C,
     "d[2 * Ln + at] = mulmod(a1[at], b1[at], q);", "d[2 * Ln + at] = mulmod(a1[at], b0[at], q);", 0,
     "test_rotation_and_relin_config3_params"),
    ("relinearisation drops the second key-switch output", C,
     "c[Ln + at] = addmod(d[Ln + at], ks[Ln + at], mods[i]);", "c[Ln + at] = d[Ln + at];", 0,
     "test_rotation_and_relin_config3_params"),
    ("BSGS giant step rotates by g instead of bb*g", C,
     "u64 gal = galois_power((u64)bb * g, n);", "u64 gal = galois_power((u64)g, n);", 0,
     "test_bsgs_banded_matvec"),
    ("BSGS plaintext diagonals transposed", C,
     "diags + ((size_t)g * bb + r) * Ln;", "diags + ((size_t)r * gg + g) * Ln;", 0,
     "test_bsgs_banded_matvec"),
    ("BSGS baby step rotation off by one", C,
     "galb[r - 1] = galois_power((u64)r, n);", "galb[r - 1] = galois_power((u64)r - 1, n);", 0,
     "test_bsgs_banded_matvec"),
    ("key generation puts P on the next digit's first limb", C,
     "if (t >= lo && t < hi) {\n                gj = 1;", "if (t >= lo && t <= hi) {\n                gj = 1;", 0,
     "test_rotation_decrypts_to_slot_rotation_config1"),
    ("key generation sign of a*s", C,
     "u64 bv = submod(e_ntt[at], mulmod(av, s_ntt[at], q), q);",
     "u64 bv = addmod(e_ntt[at], mulmod(av, s_ntt[at], q), q);", 0,
     "test_rotation_decrypts_to_slot_rotation_config1"),
    ("encryption sign of a*s", C,
     "u64 v = submod(e_ntt[at], mulmod(a[at], s_ntt[at], q), q);",
     "u64 v = addmod(e_ntt[at], mulmod(a[at], s_ntt[at], q), q);", 0,
     "test_rotation_decrypts_to_slot_rotation_config1"),
    ("Galois secret built with the wrong element", C,
     "oracle_automorph_coeff(tmp, out + (size_t)l * n, mods[l], n, g);",
     "oracle_automorph_coeff(tmp, out + (size_t)l * n, mods[l], n, (g * g) % (2 * (u64)n));", 0,
     "test_rotation_decrypts_to_slot_rotation_config1"),
    ("schoolbook product wraps cyclically", C,
     "else out[k - n] = submod(out[k - n], p, q);", "else out[k - n] = addmod(out[k - n], p, q);", 0,
     "test_negacyclic_schoolbook_tiny"),
    ("encoder conjugates the slots", "encoding.py",
     "idx = _angle_matrix(n, -1)", "idx = _angle_matrix(n, 1)", 0,
     "test_encode_decode_roundtrip_and_rotation"),
    ("modular addition wraps one too high", C,
     "static u64 addmod(u64 a, u64 b, u64 q) { return (a + b) % q; }",
     "static u64 addmod(u64 a, u64 b, u64 q) { u64 s = a + b; return s >= q ? s - q + 1 : s; }", 0,
     "test_fast_ntt_equals_definition"),
    ("monomial product never negates", C,
     "out[t] = neg ? submod(0, in[j], q) : in[j] % q;", "out[t] = in[j] % q;", 0,
     "test_mul_monomial_on_monomials"),
    ("modraise without centring", C,
     "if (d[i] != hd[i]) { neg = d[i] > hd[i]; break; }", "if (d[i] != hd[i]) { neg = 0; break; }", 0,
     "test_modraise_is_the_centred_crt_lift"),
    ("modraise centres (Q-1)/2 itself", C,
     "int neg = 0;\n            for (int i = l - 1;", "int neg = 1;\n            for (int i = l - 1;", 0,
     "test_modraise_is_the_centred_crt_lift"),
    ("modraise Garner digit with the first inverse only", C,
     "t = mulmod(submod(t, d[j] % mods[i], mods[i]), inv[(size_t)i * l + j], mods[i]);",
     "t = mulmod(submod(t, d[j] % mods[i], mods[i]), inv[(size_t)i * l], mods[i]);", 0,
     "test_modraise_is_the_centred_crt_lift"),
    ("modraise Horner from the wrong end", C,
     "for (int i = l - 1; i >= 0; --i)\n                    r = addmod(",
     "for (int i = 0; i < l; ++i)\n                    r = addmod(", 0,
     "test_modraise_is_the_centred_crt_lift"),
    ("conj_extract: imaginary part with the wrong sign", C,
     "dif[at] = submod(cj[at], c[at], q);", "dif[at] = submod(c[at], cj[at], q);", 0,
     "test_conj_extract_gives_real_and_imaginary_parts"),
    ("conj_extract with the wrong Galois element", C,
     "const u64 g = 2 * (u64)n - 1;", "const u64 g = (u64)n - 1;", 0,
     "test_conj_extract_gives_real_and_imaginary_parts"),
    ("restore_merge multiplies by -i", C,
     "mods, L, 1, n, n / 2);", "mods, L, 1, n, 3 * n / 2);", 1,
     "test_restore_merge_and_round_trip"),
    ("embedding matrix transposed", "encoding.py",
     "idx = np.outer(e, k) % (2 * n)", "idx = np.outer(k, e) % (2 * n)", 0,
     "test_embedding_matrix_rows_are_orthogonal"),
    ("coeff_to_slot matrix without the conjugate", "encoding.py",
     "return (2.0 / n) * embedding_matrix(n).conj().T", "return (2.0 / n) * embedding_matrix(n).T", 0,
     "test_embedding_matrix_rows_are_orthogonal"),
    ("BSGS plaintexts pre-rotated the wrong way", "encoding.py",
     "encode_ntt(np.roll(diag, bb * g), mods, scale, n)", "encode_ntt(np.roll(diag, -bb * g), mods, scale, n)", 0,
     "test_coeff_to_slot_gives_the_coefficients_as_slots"),
    ("sin_fold: Taylor series of cosh instead of cos", "boot.py",
     "a_k = (-1) ** k / math.factorial(2 * k)", "a_k = 1 / math.factorial(2 * k)", 0,
     "test_sin_fold_is_sine_of_two_pi_x"),
    ("sin_fold: double-angle step without the factor 2", "boot.py",
     "        c = mul_int(c, 2, chain)\n", "", 0,
     "test_sin_fold_is_sine_of_two_pi_x"),
    ("sin_fold: quarter-turn shift the wrong way", "boot.py",
     "th = add_const(th, -w / 4, s_th, chain)", "th = add_const(th, w / 4, s_th, chain)", 0,
     "test_sin_fold_is_sine_of_two_pi_x"),
    ("constants added to c1 instead of c0", "boot.py",
     'out[0] = core.pointwise("add", ct[0], c, chain.mods[:l])',
     'out[1] = core.pointwise("add", ct[1], c, chain.mods[:l])', 0,
     "test_sin_fold_is_sine_of_two_pi_x"),
    ("coeff_to_slot without the 1/2 that conj_extract doubles", "boot.py",
     "lintrans_plaintexts(0.5 * coeff_to_slot_matrix(n)", "lintrans_plaintexts(coeff_to_slot_matrix(n)", 0,
     "test_bootstrap_removes_the_multiple_of_q0"),
    ("slot_to_coeff factor q0 / (pi Delta)", "boot.py",
     "f = q0 / (2 * math.pi * delta)", "f = q0 / (math.pi * delta)", 0,
     "test_bootstrap_removes_the_multiple_of_q0"),
    ("butterfly twiddles from the (2 len)-th root", "encoding.py",
     "ang = 2 * _PI * e.astype(np.longdouble) / np.longdouble(4 * ln)",
     "ang = 2 * _PI * e.astype(np.longdouble) / np.longdouble(2 * ln)", 0,
     "test_special_fft_factorization"),
    ("inverse butterfly multiplies by D instead of D^-1", "encoding.py",
     "dm[~top], d0[~top] = 0.5 / D[j[~top]], -0.5 / D[j[~top]]",
     "dm[~top], d0[~top] = 0.5 * D[j[~top]], -0.5 * D[j[~top]]", 0,
     "test_special_fft_factorization"),
    ("diagonal product shifts the wrong way", "encoding.py",
     "out[k] = out.get(k, 0) + da * np.roll(db, -a)", "out[k] = out.get(k, 0) + da * np.roll(db, a)", 0,
     "test_special_fft_factorization"),
    ("bit reversal left out", "encoding.py",
     'int(format(i, "0%db" % bits)[::-1], 2)', 'int(format(i, "0%db" % bits), 2)', 0,
     "test_special_fft_factorization"),
    ("planned BSGS plaintexts pre-rotated the wrong way", "encoding.py",
     "encode_ntt(np.roll(d, G), mods, scale, n)", "encode_ntt(np.roll(d, -G), mods, scale, n)", 0,
     "test_factored_transforms_decrypt"),
    ("batch encoder: imaginary part added instead of subtracted", "encoding.py",
     "re = re - np.sin(ang) @ Z.imag.T", "re = re + np.sin(ang) @ Z.imag.T", 0,
     "test_batch_encoder_matches_encode_and_decodes"),
    ("batch encoder without the 2/n factor", "encoding.py",
     "v = (np.longdouble(2) / np.longdouble(n)) * re * np.longdouble(scale)",
     "v = re * np.longdouble(scale)", 0,
     "test_batch_encoder_matches_encode_and_decodes"),
    ("batch encoder: residues of the wrong prime", "encoding.py",
     "res = np.mod(m[c:c + 64, None, :], q[None, :, None])", "res = np.mod(m[c:c + 64, None, :], q[None, ::-1, None])",
     0, "test_batch_encoder_matches_encode_and_decodes"),
]


def plant(index, dest):
    """Copy oracle/ into dest with slip `index` applied; returns the copy's path."""
    name, fname, old, new, occ, _ = MUTATIONS[index]
    copy = os.path.join(dest, "oracle")
    shutil.copytree(os.path.join(ROOT, "oracle"), copy,
                    ignore=shutil.ignore_patterns("*.so", "__pycache__"))
    path = os.path.join(copy, fname)
    with open(path) as f:
        text = f.read()
    parts = text.split(old)
    if len(parts) <= occ + 1:
        raise ValueError("slip %r: text not found in %s" % (name, fname))
    text = old.join(parts[:occ + 1]) + new + old.join(parts[occ + 1:])
    with open(path, "w") as f:
        f.write(text)
    return copy


def run(index, targeted=False, timeout=1800, threads=None):
    """Run the pins against a copy with slip `index`; return (caught, first failure)."""
    env = dict(os.environ)
    if threads:
        env["OMP_NUM_THREADS"] = str(threads)
    with tempfile.TemporaryDirectory(prefix="oracle_slip_") as d:
        plant(index, d)
        cmd = [sys.executable, "-m", "pytest", *PINS, "-x", "-q", "--import-mode=append",
               "-p", "no:cacheprovider"]
        if targeted:
            cmd += ["-k", MUTATIONS[index][5]]
        # `python -m pytest` puts its working directory first on sys.path, so
        # `import oracle` finds the planted copy ahead of the repository's one
        r = subprocess.run(cmd, cwd=d, capture_output=True, text=True, timeout=timeout, env=env)
    failed = [ln.split("::")[-1].split(" - ")[0] for ln in r.stdout.splitlines()
              if ln.startswith(("FAILED", "ERROR"))]
    return r.returncode != 0, (failed[0] if failed else "")


def main(argv):
    from concurrent.futures import ThreadPoolExecutor

    targeted = "--targeted" in argv
    jobs = 1
    if "--jobs" in argv:
        k = argv.index("--jobs")
        jobs = int(argv[k + 1])
        argv = argv[:k] + argv[k + 2:]
    picks = [int(a) for a in argv if not a.startswith("--")] or list(range(len(MUTATIONS)))
    threads = max(1, (os.cpu_count() or 1) // jobs) if jobs > 1 else None
    missed = 0
    with ThreadPoolExecutor(max_workers=jobs) as pool:
        results = pool.map(lambda i: (i, run(i, targeted, threads=threads)), picks)
        for i, (caught, first) in results:
            missed += not caught
            print("%2d  %-7s %-55s %s" % (i, "caught" if caught else "MISSED", MUTATIONS[i][0],
                                          first), flush=True)
    return 1 if missed else 0


if __name__ == "__main__":
    sys.exit(main(sys.argv[1:]))
