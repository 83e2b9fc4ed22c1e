"""CPU oracle for the LSA hot path. Test infrastructure only: see lsa_ref.py."""
