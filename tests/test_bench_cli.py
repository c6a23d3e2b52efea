"""Command-line checks of bench.py that need no GPU: the profiling options
parse, and --heads is refused outside a --profile-call run (it would change
the workload the bench line names)."""
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run(*args):
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True, text=True,
                          timeout=120)


def test_help_lists_profile_options():
    r = run("--help")
    assert r.returncode == 0
    assert "--profile-call" in r.stdout and "--heads" in r.stdout


def test_heads_needs_profile_call():
    r = run("--heads", "8")
    assert r.returncode == 2
    assert "--heads only sizes --profile-call runs" in r.stderr
